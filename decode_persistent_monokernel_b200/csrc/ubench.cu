// Micro-benchmarks that bound the decode kernel's design choices on this GPU:
//   * launch overhead of back-to-back empty kernels (what a kernel-per-op
//     decode pays per launch; the monokernel page puts it near 4.5 us);
//   * the weight stream alone: the decode kernel's bulk-copy ring (one
//     producer warp, 16 consumer warps waiting on every tile), with and
//     without the consumers' dot products, from HBM or from L2;
//   * one dependency point across SMs: release-add on a counter by every CTA,
//     acquire-poll until all have arrived (the decode kernel's grid-wide
//     wait), back to back.
// Every wait here is bounded by a cycle-count watchdog that records an error
// and returns; nothing in this file spins without a limit.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kie_ubench.h"

namespace {

constexpr int kWarps = 16;              // consumer warps, as in the decode kernel
constexpr int kSlot = 32768;            // bytes per ring slot
constexpr long long kLimit = 4000000000ll;  // SM cycles before a wait gives up (~2 s)

__device__ __forceinline__ uint32_t su32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint64_t *b, uint32_t c) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(c) : "memory");
}
__device__ __forceinline__ void bar_expect(uint64_t *b, uint32_t n) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(n)
               : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool bar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ bool bar_wait(uint64_t *b, uint32_t parity, int *err) {
  const long long t0 = clock64();
  while (!bar_test(b, parity))
    if (clock64() - t0 > kLimit) {
      atomicExch(err, 1);
      return false;
    }
  return true;
}
__device__ __forceinline__ void copy_in(void *dst, const void *src, uint32_t n, uint64_t *b) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          su32(dst)),
      "l"(src), "r"(n), "r"(su32(b))
      : "memory");
}

__global__ void empty_kernel() {}

struct StreamArgs {
  const uint8_t *src;
  int64_t bytes_per_cta;   // region of each CTA (a multiple of kSlot)
  int32_t passes;          // times each CTA walks its region
  int32_t ring_slots;
  int32_t consume;         // 1: dot products of every tile, as a row GEMV
  float *sink;
  int *err;
};

// One CTA per SM: warp 16 lane 0 copies 32 KB tiles of the CTA's region into
// the ring; warps 0..15 wait on every tile in order and release it.
__global__ void __launch_bounds__((kWarps + 1) * 32, 1) stream_kernel(StreamArgs a) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int NS = a.ring_slots;
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + size_t(NS) * kSlot);
  uint64_t *empty = full + NS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      bar_init(&full[i], 1);
      bar_init(&empty[i], kWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint8_t *base = a.src + size_t(blockIdx.x) * size_t(a.bytes_per_cta);
  const uint32_t per = uint32_t(a.bytes_per_cta / kSlot);
  const uint32_t ntiles = per * uint32_t(a.passes);
  if (warp == kWarps) {
    if (lane == 0) {
      uint32_t T = 0;
      for (; T < ntiles; ++T) {
        const uint32_t s = T % NS;
        if (T >= uint32_t(NS) && !bar_wait(&empty[s], ((T / NS) - 1) & 1, a.err)) break;
        bar_expect(&full[s], kSlot);
        copy_in(sm + size_t(s) * kSlot, base + size_t(T % per) * kSlot, kSlot, &full[s]);
      }
      // every copy in flight lands before the CTA may exit
      const uint32_t first = T > uint32_t(NS) ? T - NS : 0;
      for (uint32_t t = first; t < T; ++t) bar_wait(&full[t % NS], (t / NS) & 1, a.err);
    }
    __syncwarp();
  } else {
    // row GEMV layout of the decode kernel: 8 rows of 2048 fp16 per tile,
    // two column halves per row, 64 bytes per lane
    const int rg = warp >> 1, half = warp & 1;
    float x[4][8];
    uint32_t off[4];
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      off[i] = uint32_t(rg * 2048 + (half * 128 + c) * 8) * 2u;
      for (int e = 0; e < 8; ++e) x[i][e] = 1.0f / float(1 + c + e);
    }
    uint32_t slot = 0, phase = 0;
    float tot = 0.f;
    for (uint32_t T = 0; T < ntiles; ++T) {
      int got = 1;
      if (lane == 0) got = bar_wait(&full[slot], phase, a.err);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      if (a.consume) {
        const uint8_t *tile = sm + size_t(slot) * kSlot;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 w = *reinterpret_cast<const uint4 *>(tile + off[i]);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ws[q]));
            acc = fmaf(f.x, x[i][2 * q], acc);
            acc = fmaf(f.y, x[i][2 * q + 1], acc);
          }
        }
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        tot += acc;
      }
      __syncwarp();
      if (lane == 0) bar_arrive(&empty[slot]);
      if (++slot == uint32_t(NS)) {
        slot = 0;
        phase ^= 1u;
      }
    }
    if (tot == 1234.5f) a.sink[blockIdx.x] = tot;   // keeps the arithmetic alive
  }
  __syncthreads();
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// n_rounds grid-wide dependency points in a row: every CTA adds 1 to the
// counter (release), then thread 0 polls (acquire) until all CTAs of this
// round have added; the counter is never reset inside the launch.
__global__ void barrier_kernel(uint32_t *ctr, int n_rounds, int *err) {
  __shared__ int stop;
  for (int r = 1; r <= n_rounds; ++r) {
    __syncthreads();   // everyone has read `stop` of the previous round
    if (threadIdx.x == 0) {
      red_release(ctr, 1u);
      const uint32_t target = uint32_t(r) * gridDim.x;
      const long long t0 = clock64();
      while (ld_acquire(ctr) < target)
        if (clock64() - t0 > kLimit) {
          atomicExch(err, 1);
          break;
        }
      stop = *reinterpret_cast<volatile int *>(err);
    }
    __syncthreads();
    if (stop) return;   // the same value in every thread of the block
  }
}

int status_of(cudaError_t e) { return e == cudaSuccess ? KIE_UB_OK : KIE_UB_ERR_CUDA; }

}  // namespace

extern "C" int kie_ubench_launch_overhead(int32_t n_launches, float *us_per_launch) {
  if (n_launches < 1 || !us_per_launch) return KIE_UB_ERR_INVALID;
  cudaStream_t st;
  cudaEvent_t e0, e1;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return KIE_UB_ERR_CUDA;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  for (int i = 0; i < 16; ++i) empty_kernel<<<1, 32, 0, st>>>();   // warm-up
  cudaEventRecord(e0, st);
  for (int i = 0; i < n_launches; ++i) empty_kernel<<<1, 32, 0, st>>>();
  cudaEventRecord(e1, st);
  cudaError_t e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  *us_per_launch = ms * 1e3f / float(n_launches);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaStreamDestroy(st);
  return status_of(e == cudaSuccess ? cudaGetLastError() : e);
}

extern "C" int kie_ubench_stream(const void *src, int64_t bytes_per_cta, int32_t n_ctas,
                                 int32_t passes, int32_t ring_slots, int32_t consume,
                                 float *ms_out) {
  if (!src || !ms_out || n_ctas < 1 || passes < 1 || ring_slots < 1 || ring_slots > 6 ||
      bytes_per_cta < kSlot || bytes_per_cta % kSlot != 0 ||
      (reinterpret_cast<uintptr_t>(src) & 15u) != 0)
    return KIE_UB_ERR_INVALID;
  const size_t smem = size_t(ring_slots) * kSlot + size_t(ring_slots) * 16;
  cudaError_t e = cudaFuncSetAttribute(stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return KIE_UB_ERR_CUDA;
  int *err = nullptr;
  float *sink = nullptr;
  if (cudaMalloc(&err, 4) != cudaSuccess) return KIE_UB_ERR_CUDA;
  if (cudaMalloc(&sink, size_t(n_ctas) * 4) != cudaSuccess) {
    cudaFree(err);
    return KIE_UB_ERR_CUDA;
  }
  cudaMemset(err, 0, 4);
  StreamArgs a{static_cast<const uint8_t *>(src), bytes_per_cta, passes, ring_slots, consume,
               sink, err};
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  stream_kernel<<<n_ctas, (kWarps + 1) * 32, smem>>>(a);   // warm-up
  cudaEventRecord(e0);
  stream_kernel<<<n_ctas, (kWarps + 1) * 32, smem>>>(a);
  cudaEventRecord(e1);
  e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  int herr = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
  *ms_out = ms;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaFree(err);
  cudaFree(sink);
  if (e != cudaSuccess) return KIE_UB_ERR_CUDA;
  return herr ? KIE_UB_ERR_TIMEOUT : KIE_UB_OK;
}

extern "C" int kie_ubench_barrier(int32_t n_ctas, int32_t n_rounds, float *us_per_round) {
  if (n_ctas < 1 || n_rounds < 1 || !us_per_round) return KIE_UB_ERR_INVALID;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (n_ctas > nsm) return KIE_UB_ERR_INVALID;   // every CTA must be resident at once
  uint32_t *ctr = nullptr;
  int *err = nullptr;
  if (cudaMalloc(&ctr, 4) != cudaSuccess) return KIE_UB_ERR_CUDA;
  if (cudaMalloc(&err, 4) != cudaSuccess) {
    cudaFree(ctr);
    return KIE_UB_ERR_CUDA;
  }
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaError_t e = cudaSuccess;
  float best = 1e30f;
  for (int rep = 0; rep < 3 && e == cudaSuccess; ++rep) {
    cudaMemset(ctr, 0, 4);
    cudaMemset(err, 0, 4);
    int rounds = n_rounds;
    void *args[] = {&ctr, &rounds, &err};
    cudaEventRecord(e0);
    e = cudaLaunchCooperativeKernel(reinterpret_cast<void *>(barrier_kernel), dim3(n_ctas),
                                    dim3(128), args, 0, nullptr);
    cudaEventRecord(e1);
    if (e == cudaSuccess) e = cudaEventSynchronize(e1);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
    if (ms < best) best = ms;
  }
  int herr = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
  *us_per_round = best * 1e3f / float(n_rounds);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaFree(ctr);
  cudaFree(err);
  if (e != cudaSuccess) return KIE_UB_ERR_CUDA;
  return herr ? KIE_UB_ERR_TIMEOUT : KIE_UB_OK;
}
