// Internal interface of the prompt pass (the tensor-core GEMM prefill):
// shared by the host side (kie_api.cu) and the prompt-pass kernels
// (prefill_gemm.cu, prefill.cu).  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kie {

// One GEMM launch: C[M, N] (+)= sum_p A_p[M, K] . B[N, K]^T.
struct GemmArgs {
  int32_t M, N, K;
  int32_t parts;        // A parts (stacked in one tensor map, a_part_rows rows apart), 1..3
  int32_t stages;       // pipeline depth: gemm_stages(parts)
  int32_t a_part_rows;  // rows between consecutive A parts
  int32_t b_row0;       // first row of B inside its tensor map
  int32_t dtype;        // 0 fp16, 1 bf16 (A and B alike)
  int32_t accumulate;   // 1: C += product; 0: C = product
  float *C;
  int64_t ldc;          // C row stride in elements
  uint32_t *status;     // device error word (0 = fine)
  uint64_t watchdog_ns;
};

int gemm_stages(int parts);
size_t gemm_smem_bytes(int parts);
int gemm_tile_m();
int gemm_tile_n();
int gemm_tile_k();
cudaError_t launch_gemm(const CUtensorMap &map_a, const CUtensorMap &map_b, const GemmArgs &g,
                        cudaStream_t st);

// Elementwise and attention kernels of the prompt pass (prefill.cu).
// x: fp32 [n, d] residual stream of the n prompt rows; parts: the GEMM A
// buffer, P parts of [rows_pad, K] in the storage type.
cudaError_t launch_embed_rows(const uint16_t *embed, const int32_t *tokens, int n, int d, int dtype,
                              float *x, cudaStream_t st);
// a = RMSNorm(x) * gain (per row, over d), written as P parts whose sum is a
// (each part the storage-type rounding of what the earlier parts leave).
cudaError_t launch_norm_split(const float *x, const float *gain, int n, int d, float eps, int parts,
                              int dtype, uint16_t *out, int64_t part_stride, int64_t ld, cudaStream_t st);
// out = v split into P parts, rows of len elements (no norm).
cudaError_t launch_split(const float *v, int n, int len, int64_t ldv, int parts, int dtype, uint16_t *out,
                         int64_t part_stride, int64_t ld, cudaStream_t st);
// RoPE of the q and k rows of qkv [n, (Hq + 2 Hkv) dh] at positions pos0 + r
// (q scaled by 1/sqrt(dh) in place), k and v rounded to the cache type and
// stored at those positions; k and v in qkv are replaced by their rounded
// values.
cudaError_t launch_rope_kv(float *qkv, int n, int pos0, int Hq, int Hkv, int dh, const float2 *rope,
                           uint16_t *kcache, uint16_t *vcache, int layer, int max_seq, int dtype,
                           float attn_scale, cudaStream_t st);
// Causal attention of the n prompt rows over cache positions 0 .. pos0 + r:
// o [n, Hq dh] fp32.
cudaError_t launch_prefill_attention(const float *qkv, int n, int pos0, int Hq, int Hkv, int dh,
                                     const uint16_t *kcache, const uint16_t *vcache, int layer, int max_seq,
                                     int dtype, float *o, cudaStream_t st);
// h = silu(gate) * up for gu [n, 2F] (gate columns 0..F-1, up F..2F-1), split
// into P parts.
cudaError_t launch_swiglu_split(const float *gu, int n, int F, int parts, int dtype, uint16_t *out,
                                int64_t part_stride, int64_t ld, cudaStream_t st);
// Greedy token of one logits row: the lowest index of the largest value;
// out[0] = token, or -1 if a logit is NaN.
cudaError_t launch_argmax_row(const float *z, int V, int32_t *out, cudaStream_t st);

}  // namespace kie
