// Elementwise and attention kernels of the prompt pass (the GEMM prefill):
// the steps between the tensor-core GEMMs of each layer, for all prompt rows
// at once.  Same arithmetic as the decode kernel: RMSNorm with eps inside the
// root, rotate-half RoPE from the fp32 cos/sin table, K (after RoPE) and V
// rounded to the cache type before they are stored and used, fp32 softmax
// and accumulation, SwiGLU.  GEMM inputs are written as a sum of storage-type
// parts (each the rounding of what the earlier parts leave), so that the
// tensor cores see the fp32 activations to within 2^-22 (fp16, two parts) or
// 2^-24 (bf16, three parts) relative.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "prefill_internal.h"

namespace kie {

namespace {

__device__ __forceinline__ float st_to_f(uint16_t b, int dtype) {
  return dtype == 0 ? __half2float(__ushort_as_half(b)) : __uint_as_float(uint32_t(b) << 16);
}
__device__ __forceinline__ uint16_t f_to_st(float v, int dtype) {
  return dtype == 0 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
// Writes v as `parts` storage-type words whose sum approximates v.
__device__ __forceinline__ void put_parts(float v, int parts, int dtype, uint16_t *out, int64_t part_stride) {
  float rem = v;
  for (int p = 0; p < parts; ++p) {
    const uint16_t b = f_to_st(rem, dtype);
    out[p * part_stride] = b;
    rem -= st_to_f(b, dtype);
  }
}

__device__ float block_sum(float v, float *red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

__global__ void embed_rows_kernel(const uint16_t *embed, const int32_t *tokens, int d, int dtype, float *x) {
  const int r = blockIdx.x;
  const uint16_t *e = embed + size_t(tokens[r]) * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) x[size_t(r) * d + i] = st_to_f(e[i], dtype);
}

__global__ void norm_split_kernel(const float *x, const float *gain, int d, float eps, int parts, int dtype,
                                  uint16_t *out, int64_t part_stride, int64_t ld) {
  __shared__ float red[32];
  const int r = blockIdx.x;
  const float *xr = x + size_t(r) * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
  const float sc = rsqrtf(block_sum(ss, red) / float(d) + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    put_parts(xr[i] * sc * gain[i], parts, dtype, out + size_t(r) * ld + i, part_stride);
}

__global__ void split_kernel(const float *v, int len, int64_t ldv, int parts, int dtype, uint16_t *out,
                             int64_t part_stride, int64_t ld) {
  const int r = blockIdx.x;
  for (int i = threadIdx.x; i < len; i += blockDim.x)
    put_parts(v[size_t(r) * ldv + i], parts, dtype, out + size_t(r) * ld + i, part_stride);
}

__global__ void rope_kv_kernel(float *qkv, int pos0, int Hq, int Hkv, int dh, const float2 *rope,
                               uint16_t *kcache, uint16_t *vcache, int layer, int max_seq, int dtype,
                               float attn_scale) {
  const int r = blockIdx.x, hh = blockIdx.y, half = dh >> 1;
  const int p = pos0 + r;
  const int ncols = (Hq + 2 * Hkv) * dh;
  float *row = qkv + size_t(r) * ncols;
  if (hh < Hq + Hkv) {   // a query head or a key head: rotate pairs (i, i + dh/2)
    float *h = row + size_t(hh) * dh;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      const float2 c = rope[size_t(p) * half + i];
      const float a = h[i], b = h[i + half];
      const float ra = a * c.x - b * c.y, rb = b * c.x + a * c.y;
      if (hh < Hq) {
        h[i] = ra * attn_scale;
        h[i + half] = rb * attn_scale;
      } else {
        const int g = hh - Hq;
        const uint16_t ba = f_to_st(ra, dtype), bb = f_to_st(rb, dtype);
        const size_t c0 = ((size_t(layer) * Hkv + g) * max_seq + p) * dh;
        kcache[c0 + i] = ba;
        kcache[c0 + i + half] = bb;
        h[i] = st_to_f(ba, dtype);
        h[i + half] = st_to_f(bb, dtype);
      }
    }
  } else {               // a value head: rounded
    const int g = hh - Hq - Hkv;
    float *h = row + size_t(hh) * dh;
    const size_t c0 = ((size_t(layer) * Hkv + g) * max_seq + p) * dh;
    for (int i = threadIdx.x; i < dh; i += blockDim.x) {
      const uint16_t b = f_to_st(h[i], dtype);
      vcache[c0 + i] = b;
      h[i] = st_to_f(b, dtype);
    }
  }
}

// Causal attention, one CTA per (query head, block of 32 prompt rows).  Key
// blocks of 64 cached positions are staged in shared memory as fp32; each
// thread keeps 8 scores of one query row (row tid / 8, keys tid % 8 + 8 u)
// and 16 output dimensions of that row; the 8 threads of a row share the
// online softmax state through shuffles.
constexpr int kQB = 32, kKB = 64, kAttnThreads = 256;

template <int DH>
__global__ void __launch_bounds__(kAttnThreads) prefill_attention_kernel(
    const float *qkv, int n, int pos0, int Hq, int Hkv, const uint16_t *kcache, const uint16_t *vcache,
    int layer, int max_seq, int dtype, float *o) {
  extern __shared__ float attn_smem[];
  float(*Qs)[DH + 1] = reinterpret_cast<float(*)[DH + 1]>(attn_smem);           // [kQB][DH + 1]
  float(*Ks)[DH + 1] = reinterpret_cast<float(*)[DH + 1]>(attn_smem + kQB * (DH + 1));  // [kKB][DH + 1]
  float(*Vs)[DH] = reinterpret_cast<float(*)[DH]>(attn_smem + (kQB + kKB) * (DH + 1));  // [kKB][DH]
  float(*Ps)[kKB] = reinterpret_cast<float(*)[kKB]>(attn_smem + (kQB + kKB) * (DH + 1) + kKB * DH);
  const int h = blockIdx.x, qb = blockIdx.y;
  const int g = h / (Hq / Hkv);
  const int ncols = (Hq + 2 * Hkv) * DH;
  const int r0 = qb * kQB;
  const int tid = threadIdx.x, row = tid >> 3, sub = tid & 7;
  constexpr int DPT = DH / 8;   // output dimensions per thread: sub + 8 v
  for (int i = tid; i < kQB * DH; i += kAttnThreads) {
    const int rr = i / DH, e = i - rr * DH;
    Qs[rr][e] = r0 + rr < n ? qkv[size_t(r0 + rr) * ncols + size_t(h) * DH + e] : 0.f;
  }
  float m = -INFINITY, lsum = 0.f, acc[DPT];
#pragma unroll
  for (int v = 0; v < DPT; ++v) acc[v] = 0.f;
  const int qpos = pos0 + r0 + row;                       // this thread's query position
  const int last = pos0 + min(r0 + kQB, n) - 1;           // the block's last query position
  const size_t cbase = (size_t(layer) * Hkv + g) * max_seq * DH;
  for (int k0 = 0; k0 <= last; k0 += kKB) {
    __syncthreads();
    for (int i = tid; i < kKB * DH; i += kAttnThreads) {
      const int j = i / DH, e = i - j * DH;
      const bool in = k0 + j <= last;
      Ks[j][e] = in ? st_to_f(kcache[cbase + size_t(k0 + j) * DH + e], dtype) : 0.f;
      Vs[j][e] = in ? st_to_f(vcache[cbase + size_t(k0 + j) * DH + e], dtype) : 0.f;
    }
    __syncthreads();
    float s[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) s[u] = 0.f;
    for (int e = 0; e < DH; ++e) {
      const float q = Qs[row][e];
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] = fmaf(q, Ks[sub + 8 * u][e], s[u]);
    }
    float mx = m;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (k0 + sub + 8 * u > qpos) s[u] = -INFINITY;    // causal mask
      mx = fmaxf(mx, s[u]);
    }
    for (int of = 4; of; of >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, of));
    const float corr = mx == -INFINITY ? 1.f : expf(m - mx);
    float ps = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float pu = s[u] == -INFINITY ? 0.f : expf(s[u] - mx);
      Ps[row][sub + 8 * u] = pu;
      ps += pu;
    }
    for (int of = 4; of; of >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, of);
    lsum = lsum * corr + ps;
    m = mx;
    __syncwarp();
#pragma unroll
    for (int v = 0; v < DPT; ++v) acc[v] *= corr;
    for (int j = 0; j < kKB; ++j) {
      const float pj = Ps[row][j];
#pragma unroll
      for (int v = 0; v < DPT; ++v) acc[v] = fmaf(pj, Vs[j][sub + 8 * v], acc[v]);
    }
  }
  if (r0 + row < n) {
    float *orow = o + size_t(r0 + row) * Hq * DH + size_t(h) * DH;
#pragma unroll
    for (int v = 0; v < DPT; ++v) orow[sub + 8 * v] = acc[v] / lsum;
  }
}

__global__ void swiglu_split_kernel(const float *gu, int F, int parts, int dtype, uint16_t *out,
                                    int64_t part_stride, int64_t ld) {
  const int r = blockIdx.x;
  const float *row = gu + size_t(r) * 2 * F;
  for (int i = threadIdx.x; i < F; i += blockDim.x) {
    const float gt = row[i], up = row[F + i];
    put_parts(gt / (1.f + expf(-gt)) * up, parts, dtype, out + size_t(r) * ld + i, part_stride);
  }
}

__global__ void argmax_row_kernel(const float *z, int V, int32_t *out) {
  __shared__ float bv[32];
  __shared__ int bi[32];
  __shared__ int nan_seen;
  if (threadIdx.x == 0) nan_seen = 0;
  __syncthreads();
  float best = -INFINITY;
  int idx = 0;
  for (int i = threadIdx.x; i < V; i += blockDim.x) {
    const float v = z[i];
    if (v != v) nan_seen = 1;
    if (v > best) { best = v; idx = i; }   // i increases: the first maximum is kept
  }
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (ov > best || (ov == best && oi < idx)) { best = ov; idx = oi; }
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) { bv[w] = best; bi[w] = idx; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < int(blockDim.x >> 5); ++i)
      if (bv[i] > best || (bv[i] == best && bi[i] < idx)) { best = bv[i]; idx = bi[i]; }
    out[0] = nan_seen ? -1 : idx;
  }
}

}  // namespace

cudaError_t launch_embed_rows(const uint16_t *embed, const int32_t *tokens, int n, int d, int dtype, float *x,
                              cudaStream_t st) {
  embed_rows_kernel<<<n, 256, 0, st>>>(embed, tokens, d, dtype, x);
  return cudaGetLastError();
}

cudaError_t launch_norm_split(const float *x, const float *gain, int n, int d, float eps, int parts, int dtype,
                              uint16_t *out, int64_t part_stride, int64_t ld, cudaStream_t st) {
  norm_split_kernel<<<n, 256, 0, st>>>(x, gain, d, eps, parts, dtype, out, part_stride, ld);
  return cudaGetLastError();
}

cudaError_t launch_split(const float *v, int n, int len, int64_t ldv, int parts, int dtype, uint16_t *out,
                         int64_t part_stride, int64_t ld, cudaStream_t st) {
  split_kernel<<<n, 256, 0, st>>>(v, len, ldv, parts, dtype, out, part_stride, ld);
  return cudaGetLastError();
}

cudaError_t launch_rope_kv(float *qkv, int n, int pos0, int Hq, int Hkv, int dh, const float2 *rope,
                           uint16_t *kcache, uint16_t *vcache, int layer, int max_seq, int dtype,
                           float attn_scale, cudaStream_t st) {
  rope_kv_kernel<<<dim3(n, Hq + 2 * Hkv), 64, 0, st>>>(qkv, pos0, Hq, Hkv, dh, rope, kcache, vcache, layer,
                                                      max_seq, dtype, attn_scale);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const float *qkv, int n, int pos0, int Hq, int Hkv, int dh,
                                     const uint16_t *kcache, const uint16_t *vcache, int layer, int max_seq,
                                     int dtype, float *o, cudaStream_t st) {
  dim3 grid(Hq, (n + kQB - 1) / kQB);
  auto smem = [](int DH) { return size_t((kQB + kKB) * (DH + 1) + kKB * DH + kQB * kKB) * 4; };
  cudaError_t e;
  if (dh == 128) {
    e = cudaFuncSetAttribute(prefill_attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem(128)));
    if (e != cudaSuccess) return e;
    prefill_attention_kernel<128><<<grid, kAttnThreads, smem(128), st>>>(qkv, n, pos0, Hq, Hkv, kcache, vcache,
                                                                         layer, max_seq, dtype, o);
  } else {
    e = cudaFuncSetAttribute(prefill_attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem(64)));
    if (e != cudaSuccess) return e;
    prefill_attention_kernel<64><<<grid, kAttnThreads, smem(64), st>>>(qkv, n, pos0, Hq, Hkv, kcache, vcache,
                                                                       layer, max_seq, dtype, o);
  }
  return cudaGetLastError();
}

cudaError_t launch_swiglu_split(const float *gu, int n, int F, int parts, int dtype, uint16_t *out,
                                int64_t part_stride, int64_t ld, cudaStream_t st) {
  swiglu_split_kernel<<<n, 256, 0, st>>>(gu, F, parts, dtype, out, part_stride, ld);
  return cudaGetLastError();
}

cudaError_t launch_argmax_row(const float *z, int V, int32_t *out, cudaStream_t st) {
  argmax_row_kernel<<<1, 1024, 0, st>>>(z, V, out);
  return cudaGetLastError();
}

}  // namespace kie
