// Tensor-core GEMM of the prompt pass (sm_100a, tcgen05):
//     C[M, N] (+)= sum_p A_p[M, K] . B[N, K]^T
// A_p: the activation matrix split into P parts of the weight type (their sum
// carries fp32-level precision), B: a weight matrix in its canonical
// row-major [out, in] layout (K-major), C: fp32 row-major.
//
// One CTA per 128 x 128 output tile.  Warp 0 (one lane) streams 64-column K
// slices of every A part and of B into a 3- or 4-stage shared-memory ring with
// tensor-map bulk copies (cp.async.bulk.tensor, 128-byte swizzle, local
// global memory only, no multicast); warp 1 allocates 512 tensor-memory
// columns and one lane issues tcgen05.mma (M 128, N 128, K 16, fp32
// accumulation in tensor memory) for each slice, handing the stage back with
// tcgen05.commit; warps 2..5 (one per tensor-memory lane quarter) read the
// result with tcgen05.ld and store or add it to C.  Four accumulators: the
// small A parts each into their own (their products would lose low-order
// bits in the aligned, truncated sums of an accumulator that holds the large
// part's products), the large part round-robin over the rest by K slice (a
// shorter chain of sequential accumulations each); the epilogue adds them in
// order with rounded fp32 adds.  Every wait is
// bounded; on expiry the CTA raises the error word and leaves after
// releasing its tensor memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "prefill_internal.h"

namespace kie {

namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64;   // tile; kBK fp16/bf16 = 128 bytes per row
constexpr int kMaxStages = 4;
constexpr int kTileBytes = kBM * kBK * 2;        // one 128 x 64 operand tile: 16 KB
constexpr int kGemmThreads = 192;                // 6 warps
constexpr int kAcc = 4;                          // tensor-memory accumulators of 128 columns

__device__ __forceinline__ uint32_t su32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint64_t *b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_expect(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_try(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a barrier phase; false (and the error word set) on expiry.
__device__ bool bar_wait(uint64_t *b, uint32_t parity, const GemmArgs &g, uint32_t code) {
  if (bar_try(b, parity)) return true;
  const long long t0 = clock64(), limit = (long long)g.watchdog_ns * 2;
  while (!bar_try(b, parity)) {
    if (clock64() - t0 > limit) {
      atomicCAS(g.status, 0u, code);
      return false;
    }
    if (*(volatile uint32_t *)g.status) return false;   // another CTA gave up
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(su32(bar))
      : "memory");
}
// Shared-memory matrix descriptor of a K-major tile stored as 128-byte
// swizzled rows (what the tensor map writes): 8-row groups 1024 bytes apart
// (stride offset), leading offset 16 bytes (unused for swizzled K-major),
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

}  // namespace

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, A and B
// both fp16 (dtype 0) or both bf16 (dtype 1), both K-major, M 128, N 128.
static __host__ __device__ uint32_t gemm_idesc(int dtype) {
  return (1u << 4) | (uint32_t(dtype) << 7) | (uint32_t(dtype) << 10) | (uint32_t(kBN >> 3) << 17) |
         (uint32_t(kBM >> 4) << 24);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const GemmArgs g) {
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  // 1024-byte aligned stages: [P A tiles][B tile] per stage
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = (g.parts + 1) * kTileBytes;
  const int kStages = g.stages;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + size_t(kStages) * stage_bytes);
  uint64_t *empty = full + kMaxStages;
  uint64_t *done = empty + kMaxStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int nk = (g.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    bar_init(done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {   // kAcc accumulators of 128 fp32 columns x 128 lanes
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(128 * kAcc)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer: K slice kt of every A part and of B into stage kt % kStages
    const uint32_t bytes = uint32_t(g.parts + 1) * kTileBytes;
    for (int kt = 0; kt < nk; ++kt) {
      const int s = kt % kStages;
      if (kt >= kStages && !bar_wait(&empty[s], ((kt / kStages) - 1) & 1, g, 0x101u)) break;
      uint8_t *st = base + size_t(s) * stage_bytes;
      bar_expect(&full[s], bytes);
      for (int p = 0; p < g.parts; ++p)
        tma_load_2d(st + size_t(p) * kTileBytes, &map_a, kt * kBK, p * g.a_part_rows + m0, &full[s]);
      tma_load_2d(st + size_t(g.parts) * kTileBytes, &map_b, kt * kBK, g.b_row0 + n0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer: 4 K16 steps per part per slice into the tensor-memory accumulator
    const uint32_t idesc = gemm_idesc(g.dtype);
    bool ok = true;
    for (int kt = 0; kt < nk && ok; ++kt) {
      const int s = kt % kStages;
      ok = bar_wait(&full[s], (kt / kStages) & 1, g, 0x102u);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t st = su32(base + size_t(s) * stage_bytes);
      const uint64_t bdesc = sw128_desc(st + uint32_t(g.parts) * kTileBytes);
      // part 0 of slice kt accumulates into accumulator kt % c0, part p > 0
      // into accumulator c0 + p - 1 (c0 = kAcc - parts + 1); each
      // accumulator's first product overwrites it
      const int c0 = kAcc - g.parts + 1;
      for (int p = 0; p < g.parts; ++p) {
        const uint64_t adesc = sw128_desc(st + uint32_t(p) * kTileBytes);
        const int ai = p == 0 ? kt % c0 : c0 + p - 1;
        const bool fresh = p == 0 ? kt < c0 : kt == 0;
        const uint32_t acc = tmem + uint32_t(ai * kBN);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)   // 16 elements = 32 bytes = 2 descriptor units
          mma_f16(acc, adesc + uint64_t(2 * k), bdesc + uint64_t(2 * k), idesc,
                  (!fresh || k > 0) ? 1u : 0u);
      }
      mma_commit(&empty[s]);   // the stage is free once these MMAs have read it
    }
    mma_commit(done);          // the accumulator is complete once every MMA has
  } else if (warp >= 2) {
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 = tile rows
    const int q = warp & 3;
    const bool ok = bar_wait(done, 0, g, 0x103u);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const int row = m0 + 32 * q + lane;
    // accumulators that received products: part 0's first min(c0, nk), then
    // one per further part
    const int cz = kAcc - g.parts + 1;
    const int n0acc = min(cz, nk);
    for (int c0 = 0; c0 < kBN && ok; c0 += 32) {
      // the accumulators added in order, with rounded fp32 adds: part 0's,
      // then the smaller parts'
      float sum[32];
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(c0), r);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int j = 0; j < 32; ++j) sum[j] = __uint_as_float(r[j]);
      for (int i = 1; i < n0acc + g.parts - 1; ++i) {
        const int a = i < n0acc ? i : cz + (i - n0acc);
        tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(a * kBN + c0), r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 32; ++j) sum[j] += __uint_as_float(r[j]);
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(sum[j]);
      if (row < g.M) {
        float *crow = g.C + size_t(row) * g.ldc + n0 + c0;
        const int ncol = min(32, g.N - (n0 + c0));
        if (ncol == 32 && (g.ldc & 3) == 0) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 v = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                   __uint_as_float(r[j + 3]));
            float4 *dst = reinterpret_cast<float4 *>(crow + j);
            if (g.accumulate) {
              const float4 o = *dst;
              v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
            }
            *dst = v;
          }
        } else {
          for (int j = 0; j < ncol; ++j) {
            const float v = __uint_as_float(r[j]);
            crow[j] = g.accumulate ? crow[j] + v : v;
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128 * kAcc)
                 : "memory");
  }
}

// Pipeline depth: four stages, or three when the A operand has three parts.
int gemm_stages(int parts) { return parts >= 3 ? 3 : kMaxStages; }
size_t gemm_smem_bytes(int parts) {
  return size_t(gemm_stages(parts)) * (parts + 1) * kTileBytes + 1024 + 256;
}

int gemm_tile_m() { return kBM; }
int gemm_tile_n() { return kBN; }
int gemm_tile_k() { return kBK; }

cudaError_t launch_gemm(const CUtensorMap &map_a, const CUtensorMap &map_b, const GemmArgs &g,
                        cudaStream_t st) {
  if (g.parts < 1 || g.parts > 3 || g.stages != gemm_stages(g.parts)) return cudaErrorInvalidValue;
  const size_t smem = gemm_smem_bytes(g.parts);
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((g.N + kBN - 1) / kBN, (g.M + kBM - 1) / kBM);
  gemm_tc_kernel<<<grid, kGemmThreads, smem, st>>>(map_a, map_b, g);
  return cudaGetLastError();
}

}  // namespace kie
