// msda_proj.cu -- the output projection after the MSDeformAttn core on the
// 5th-generation tensor cores (sm_100a: TMA bulk tensor loads, tcgen05.mma with
// the accumulator in tensor memory).
//
// "Deformable DETR模型解读（附源码+论文）", MultiScaleDeformableAttention.forward:
// the core's output [N, Lq, M*D] goes through output_proj, a Linear layer:
//     Y[r, n] = sum_k X[r, k] * Wt[n, k] + bias[n]      (Wt: [C_out, C_in])
// This is a dense contraction, so it runs on the tensor cores: kind::tf32
// (float32 operands read as TF32, float32 accumulation).
//
// One persistent CTA per SM walks row tiles of 128 rows; K is cut into chunks of
// 32 (one 128-byte row of float32).  The CTA's chunks form one sequence g = 0,
// 1, ... (tile-major) that flows through a ring of kProjStages shared-memory
// stages.  Roles, one warp each, synchronised by mbarriers only:
//   warp 0 (one lane)  TMA producer: loads the X box [128 rows x 32] and the Wt
//                      box [C_out x 32] of chunk g into stage g % kProjStages
//                      with 128-byte swizzle, once the MMAs of chunk
//                      g - kProjStages have released that stage.
//   warp 1 (one lane)  MMA issuer: per chunk four M=128 x N=C_out x K=8 MMAs into
//                      the tile's accumulator, committed to the stage's "empty"
//                      barrier; after a tile's last chunk a commit to the
//                      accumulator's "full" barrier.
//   warps 4..7         epilogue: warp 4 + q reads accumulator lanes (rows)
//                      32 q .. 32 q + 31 with tcgen05.ld, adds the bias, writes
//                      the rows and releases the accumulator.
// Two accumulators (2 x 256 of the SM's 512 tensor-memory columns) alternate
// between tiles, so a tile's epilogue overlaps the next tile's loads and MMAs.
//
// Precise mode (PRECISE, msda_output_projection_f32): float32 accuracy from
// three TF32 products.  Each operand is split into a TF32 head and a float32
// remainder, x = hi + lo with hi = x with its 13 low mantissa bits cleared (so
// x - hi is exact in float32 and |lo| < 2^-10 |x|), and
//     x w ~ hi_x hi_w + hi_x lo_w + lo_x hi_w,
// dropping lo_x lo_w (< 2^-20 |x w|); lo read as TF32 loses < 2^-10 |lo|.  Two
// more warps do the split: the CTA has 384 threads, and warps 2..3 and 8..11 wait
// for a stage's copies, rewrite its X and W elements as their heads in place and
// write the remainders into a second buffer of the stage at the same (swizzled)
// offsets, then arrive on the stage's "split" barrier, which the MMA issuer
// waits for instead of "full".  The
// heads are written back explicitly so that the split is exact whether the
// tensor cores truncate or round a TF32 operand.  A stage then holds the four
// operand buffers (96 KB), so two stages fit.
// TMA fills rows and K columns past the end with zeros.  Every wait is bounded
// in time: past the limit the waiting thread sets a flag that stops every role;
// the CTA then waits (bounded again) for its copies and MMAs in flight, releases
// its tensor memory and reports the failure to the host through a device flag
// (msda_output_projection_check).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kProjThreads = 256;
constexpr int kProjRows = 128;                                  // MMA M: rows per tile
constexpr int kProjChunk = 32;                                  // K per stage (128 bytes)
constexpr int kProjStages = 4;
constexpr int kProjMaxOut = 256;                                // MMA N limit
constexpr int kProjXBytes = kProjRows * kProjChunk * 4;         // 16 KB
constexpr int kProjStageBytes = kProjXBytes + kProjMaxOut * kProjChunk * 4;  // 48 KB
// Epilogue staging: per epilogue warp two buffers of 32 rows x 32 floats (4 KB,
// 128-byte swizzle) that TMA stores to Y.
constexpr int kProjOutBytes = 32 * 32 * 4;
constexpr int kProjOutOffset = kProjStages * kProjStageBytes;
constexpr int kProjSmemBytes = kProjOutOffset + 4 * 2 * kProjOutBytes + 1024;  // + alignment
// Precise mode: two stages of X, W heads then X, W remainders.
constexpr int kPreciseStages = 2;
constexpr int kPreciseStageBytes = 2 * kProjStageBytes;  // 96 KB
constexpr int kPreciseOutOffset = kPreciseStages * kPreciseStageBytes;
constexpr int kPreciseSmemBytes = kPreciseOutOffset + 4 * 2 * kProjOutBytes + 1024;
constexpr int kPreciseThreads = 384;
constexpr int kSplitThreads = 192;  // warps 2..3 and 8..11
constexpr uint32_t kAccColumns = 256;                           // per accumulator
constexpr unsigned long long kProjWaitNs = 1000000000ull;       // 1 s per wait

struct ProjBarriers {
  uint64_t full[kProjStages];   // the TMA bytes of a stage have landed
  uint64_t empty[kProjStages];  // the MMAs reading a stage are done
  uint64_t acc_full[2];         // an accumulator holds a finished tile
  uint64_t acc_empty[2];        // the 4 epilogue warps have read an accumulator
  uint64_t drain;               // every MMA issued has finished (failure path)
  uint64_t split[kProjStages];  // precise mode: a stage's heads and remainders are written
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits until the phase of `bar` with the given parity has completed.  Gives
// up when another role has set *failed (if `stop` is non-null) or after
// kProjWaitNs, setting *failed itself.
__device__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* failed,
                             volatile int* stop) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned polls = 1;; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if (stop != nullptr && *stop) return false;
    if ((polls & 255u) == 0 && global_ns() - t0 > kProjWaitNs) {
      *failed = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %0;" ::"r"(bytes),
               "r"(smem_u32(bar))
               : "memory");
}

// 2-D TMA tile load of the box at element coordinates (x innermost, y) into
// shared memory, completing on `bar`.  x is always a multiple of 32 floats.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 2-D TMA tile store of a shared-memory box to element coordinates (x, y) of
// the tensor; elements past the tensor's end are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// D (tensor memory) [+]= A * B, kind::tf32, operands from shared-memory descriptors.
__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      :
      : "r"(d), "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Matrix descriptor of a K-major operand that TMA wrote with 128-byte swizzle:
// one 128-byte row per M (or N) index, 8-row swizzle atoms 1024 bytes apart
// (SBO), LBO unused (1), descriptor version 1, layout SWIZZLE_128B.  The stage
// bases are 1024-byte aligned, so the base-offset field stays 0; the K step k of
// a chunk starts 32 k bytes into each row.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t start) {
  return static_cast<uint64_t>((start >> 4) & 0x3fff) | (1ull << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::tf32: D float32, A and B TF32, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t tf32_idesc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kProjRows >> 4) << 24);
}

// The TF32 head of x: its 13 low mantissa bits cleared (x itself if not finite).
__device__ __forceinline__ float tf32_head(float x) {
  return isfinite(x) ? __int_as_float(__float_as_int(x) & static_cast<int>(0xffffe000u)) : x;
}

template <bool PRECISE>
__global__ void __launch_bounds__(PRECISE ? kPreciseThreads : kProjThreads, 1)
proj_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
            const __grid_constant__ CUtensorMap tmap_y, const float* __restrict__ bias,
            long long rows, int c_in, int c_out, int* __restrict__ status) {
  constexpr int STAGES = PRECISE ? kPreciseStages : kProjStages;
  constexpr int STAGE_BYTES = PRECISE ? kPreciseStageBytes : kProjStageBytes;
  constexpr int OUT_OFFSET = PRECISE ? kPreciseOutOffset : kProjOutOffset;
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) ProjBarriers bars;
  __shared__ uint32_t tmem_base;
  __shared__ int failed_flag;
  volatile int* failed = &failed_flag;

  // The swizzled stages need 1024-byte alignment.
  const uint32_t stages = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(2 * kAccColumns));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 32) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
      if (PRECISE) mbar_init(&bars.split[s], kSplitThreads);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars.acc_full[a], 1);
      mbar_init(&bars.acc_empty[a], 4);
    }
    mbar_init(&bars.drain, 1);
    failed_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;

  const long long tiles = (rows + kProjRows - 1) / kProjRows;
  const long long my_tiles =
      blockIdx.x < tiles ? (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int nch = (c_in + kProjChunk - 1) / kProjChunk;
  const long long total = my_tiles * nch;  // chunks of this CTA

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer -------------------------------------------------------
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x))
                   : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w))
                   : "memory");
      const uint32_t stage_tx = static_cast<uint32_t>(kProjXBytes + c_out * kProjChunk * 4);
      long long issued = 0;
      bool ok = true;
      for (long long g = 0; g < total; ++g) {
        const int s = static_cast<int>(g % STAGES);
        // Stage s was last read by the MMAs of chunk g - STAGES.
        if (g >= STAGES &&
            !wait_bounded(&bars.empty[s], static_cast<uint32_t>((g / STAGES - 1) & 1),
                          failed, failed)) {
          ok = false;
          break;
        }
        const long long tile = blockIdx.x + (g / nch) * gridDim.x;
        const int k0 = static_cast<int>(g % nch) * kProjChunk;
        const uint32_t st = stages + static_cast<uint32_t>(s * STAGE_BYTES);
        mbar_expect_tx(&bars.full[s], stage_tx);
        tma_load_2d(st, &tmap_x, k0, static_cast<int>(tile * kProjRows), &bars.full[s]);
        tma_load_2d(st + kProjXBytes, &tmap_w, k0, 0, &bars.full[s]);
        issued = g + 1;
      }
      // Every copy issued lands before the CTA exits (a stage's earlier chunks
      // were consumed before it was refilled, so only the last ones can be in
      // flight).  Then, on the normal path, wait for each stage's last MMA
      // commit, so that no MMA still reads shared memory and no arrival is
      // pending at exit.
      const long long first = issued > STAGES ? issued - STAGES : 0;
      for (long long g = first; g < issued; ++g)
        wait_bounded(&bars.full[g % STAGES], static_cast<uint32_t>((g / STAGES) & 1), failed,
                     nullptr);
      if (ok)
        for (long long g = first; g < issued; ++g)
          wait_bounded(&bars.empty[g % STAGES], static_cast<uint32_t>((g / STAGES) & 1), failed,
                       failed);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ---------------------------------------------------------
      const uint32_t idesc = tf32_idesc(c_out);
      bool ok = true;
      long long g = 0;
      for (long long lt = 0; lt < my_tiles && ok; ++lt) {
        const int acc = static_cast<int>(lt & 1);
        // The epilogue of tile lt - 2 must have read this accumulator.
        if (lt >= 2 && !wait_bounded(&bars.acc_empty[acc],
                                     static_cast<uint32_t>((lt / 2 - 1) & 1), failed, failed)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d = tmem + static_cast<uint32_t>(acc) * kAccColumns;
        for (int c = 0; c < nch; ++c, ++g) {
          const int s = static_cast<int>(g % STAGES);
          // Plain mode: the stage's copies have landed.  Precise mode: its
          // heads and remainders have been written.
          uint64_t* ready = PRECISE ? &bars.split[s] : &bars.full[s];
          if (!wait_bounded(ready, static_cast<uint32_t>((g / STAGES) & 1), failed, failed)) {
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t xa = stages + static_cast<uint32_t>(s * STAGE_BYTES);
          const uint32_t wa = xa + kProjXBytes;
          const int ksteps = min(kProjChunk, c_in - c * kProjChunk) / 8;
          for (int k = 0; k < ksteps; ++k) {
            const uint64_t da = sw128_desc(xa + 32 * k);
            const uint64_t db = sw128_desc(wa + 32 * k);
            const uint32_t accumulate = (c > 0 || k > 0) ? 1u : 0u;
            mma_tf32(d, da, db, idesc, accumulate);
            if constexpr (PRECISE) {
              // hi_x lo_w + lo_x hi_w (the remainders sit kProjStageBytes on).
              mma_tf32(d, da, sw128_desc(wa + kProjStageBytes + 32 * k), idesc, 1u);
              mma_tf32(d, sw128_desc(xa + kProjStageBytes + 32 * k), db, idesc, 1u);
            }
          }
          mma_commit(&bars.empty[s]);
        }
        if (ok) mma_commit(&bars.acc_full[acc]);
      }
      if (!ok) {
        // Failure: every MMA issued finishes before the tensor memory is freed.
        mma_commit(&bars.drain);
        wait_bounded(&bars.drain, 0u, failed, nullptr);
      }
    }
    __syncwarp();
  } else if (PRECISE && (warp == 2 || warp == 3 || warp >= 8)) {
    // ---- splitter (precise mode) --------------------------------------------
    const int t = warp < 8 ? tid - 64 : tid - 256 + 64;
    const int n16 = (kProjXBytes + c_out * kProjChunk * 4) / 16;  // X then W, 16 bytes each
    for (long long g = 0; g < total; ++g) {
      const int s = static_cast<int>(g % STAGES);
      const bool ok = wait_bounded(&bars.full[s], static_cast<uint32_t>((g / STAGES) & 1),
                                   failed, failed);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint32_t hi = stages + static_cast<uint32_t>(s * STAGE_BYTES);
      const uint32_t lo = hi + kProjStageBytes;
      for (int i = t; i < n16; i += kSplitThreads) {
        float4 v;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                     : "r"(hi + 16 * i));
        const float4 h = make_float4(tf32_head(v.x), tf32_head(v.y), tf32_head(v.z),
                                     tf32_head(v.w));
        // x - hi is exact; a non-finite x keeps all of itself in the head.
        const float4 r = make_float4(isfinite(v.x) ? v.x - h.x : 0.0f,
                                     isfinite(v.y) ? v.y - h.y : 0.0f,
                                     isfinite(v.z) ? v.z - h.z : 0.0f,
                                     isfinite(v.w) ? v.w - h.w : 0.0f);
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(hi + 16 * i), "f"(h.x),
                     "f"(h.y), "f"(h.z), "f"(h.w)
                     : "memory");
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(lo + 16 * i), "f"(r.x),
                     "f"(r.y), "f"(r.z), "f"(r.w)
                     : "memory");
      }
      // The MMAs read the stage through the async proxy.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars.split[s]);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---- epilogue -------------------------------------------------------------
    const int quarter = warp - 4;  // tcgen05.ld: warp w reaches lanes 32 (w % 4) .. + 31
    if (lane == 0)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_y))
                   : "memory");
    const uint32_t out0 =
        stages + static_cast<uint32_t>(OUT_OFFSET + quarter * 2 * kProjOutBytes);
    int nbuf = 0;  // blocks this warp has staged (buffer = nbuf & 1)
    for (long long lt = 0; lt < my_tiles; ++lt) {
      const int acc = static_cast<int>(lt & 1);
      const bool ready = wait_bounded(&bars.acc_full[acc], static_cast<uint32_t>((lt / 2) & 1),
                                      failed, failed);
      if (!__all_sync(0xffffffffu, ready)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const long long tile = blockIdx.x + lt * gridDim.x;
      const int row0 = static_cast<int>(tile * kProjRows) + quarter * 32;
      const uint32_t src = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                           static_cast<uint32_t>(acc) * kAccColumns;
      for (int c0 = 0; c0 < c_out; c0 += 32, ++nbuf) {
        // This thread's row (lane) of columns c0 .. c0 + 31; past c_out the
        // values are never stored.
        uint32_t v[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
              "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
              "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(src + static_cast<uint32_t>(c0)));
        const bool two = c0 + 16 < c_out;
        if (two)
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
              "%10, %11, %12, %13, %14, %15}, [%16];"
              : "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
                "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
              : "r"(src + static_cast<uint32_t>(c0 + 16)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        // The store issued from this buffer two blocks ago has read it.
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        const uint32_t buf = out0 + static_cast<uint32_t>((nbuf & 1) * kProjOutBytes);
        // Row `lane`, 16-byte chunk q of the block goes to chunk q ^ (lane % 8)
        // (the 128-byte swizzle TMA undoes on the way out).
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q >= 4 && !two) break;
          float4 o = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
          if (bias != nullptr) {
            const float* b = bias + c0 + 4 * q;
            o.x += __ldg(b);
            o.y += __ldg(b + 1);
            o.z += __ldg(b + 2);
            o.w += __ldg(b + 3);
          }
          const uint32_t a = buf + static_cast<uint32_t>(lane * 128 + ((q ^ (lane & 7)) * 16));
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(o.x), "f"(o.y),
                       "f"(o.z), "f"(o.w)
                       : "memory");
        }
        // The writes must be visible to the bulk copy (async proxy).
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        // A box that starts past the last row has nothing to store.
        if (lane == 0 && row0 < rows) tma_store_2d(&tmap_y, buf, c0, row0);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
    }
    // Every store has completed before the CTA exits.
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (tid == 0 && *failed) atomicExch(status, 1);
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * kAccColumns));
}

// Set by a CTA whose wait ran past the limit.
__device__ int g_projection_failed;

PFN_cuTensorMapEncodeTiled encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  });
  return fn;
}

// Tensor map of a row-major float32 array [outer, inner] moved in boxes of
// [box_outer, 32] with 128-byte swizzle; loads read elements past either end as
// zero, stores skip them.
bool make_map(CUtensorMap* map, const float* base, long long inner, long long outer,
              int box_outer) {
  PFN_cuTensorMapEncodeTiled fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * sizeof(float)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kProjChunk),
                             static_cast<cuuint32_t>(box_outer)};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t projection_failed_flag(int** flag) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(flag), g_projection_failed);
}

cudaError_t launch_projection(const float* x, const float* weight, const float* bias, float* y,
                              long long rows, int c_in, int c_out, bool precise,
                              cudaStream_t stream) {
  static_assert(kProjSmemBytes <= 227 * 1024, "the stages must fit one CTA");
  static_assert(kPreciseSmemBytes + 256 <= 227 * 1024, "the precise stages must fit one CTA");
  if (rows == 0) return cudaSuccess;
  // Coordinates of the row tiles are 32-bit in the TMA instruction.
  if (rows > static_cast<long long>(INT32_MAX) - kProjRows) return cudaErrorInvalidValue;
  int* status = nullptr;
  cudaError_t err = projection_failed_flag(&status);
  if (err != cudaSuccess) return err;
  CUtensorMap map_x, map_w, map_y;
  if (!make_map(&map_x, x, c_in, rows, kProjRows) ||
      !make_map(&map_w, weight, c_in, c_out, c_out) || !make_map(&map_y, y, c_out, rows, 32))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  const auto kernel = precise ? proj_kernel<true> : proj_kernel<false>;
  const int smem = precise ? kPreciseSmemBytes : kProjSmemBytes;
  if ((err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
      cudaSuccess)
    return err;
  const long long tiles = (rows + kProjRows - 1) / kProjRows;
  const long long grid = tiles < sms ? tiles : sms;
  kernel<<<static_cast<unsigned>(grid), precise ? kPreciseThreads : kProjThreads, smem, stream>>>(
      map_x, map_w, map_y, bias, rows, c_in, c_out, status);
  return cudaGetLastError();
}

}  // namespace msda
