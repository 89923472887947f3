// The persistent batch-1 decode kernel ("monokernel": Kog Inference Engine
// write-ups, monokernel bullet -- the whole decode path as one persistent
// kernel, no launch between layers; "Software versus silicon" section --
// prefill, decode and LM-head sampling in one go, grid synchronisations and
// per-launch overhead removed).
//
// One CTA per SM, all co-resident (cooperative launch).  Each CTA has
//   * one producer warp: streams the CTA's pre-swizzled weight tiles, in the
//     order the CTA consumes them, through a ring of shared-memory slots with
//     cp.async.bulk (1-D bulk copies, no tensor map, no multicast) and
//     mbarrier completion.  Weights do not depend on activations, so the
//     producer runs ahead across stage, layer and token boundaries while the
//     consumers wait on other CTAs: HBM keeps streaming during every wait;
//   * kConsumerWarps consumer warps: stage the input vector (RMSNorm fused),
//     run the row-split GEMV tiles from shared memory, reduce, apply the
//     stage epilogue (SwiGLU, residual add, argmax), and do the split-KV
//     attention.
// Cross-CTA dependencies use monotonically increasing epoch counters in
// global memory (release add / acquire load), never a full grid barrier
// primitive.  Every spin is bounded by a %globaltimer watchdog; on expiry
// the CTA records an error, raises the abort flag and every CTA leaves
// after draining its in-flight copies.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kie_internal.h"

namespace kie {

constexpr int kNC = kConsumerWarps * 32;  // consumer threads
constexpr int kThreads = kNC + 32;        // + one producer warp

// Device error codes written to the status word (low byte: kind).
enum DevErr : uint32_t {
  DE_TIMEOUT_COUNTER = 1,
  DE_TIMEOUT_FULL = 2,
  DE_TIMEOUT_EMPTY = 3,
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// Named barrier over the consumer warps only (the producer never joins).
__device__ __forceinline__ void cbar() {
  __syncwarp();
  asm volatile("bar.sync 1, %0;" ::"n"(kNC) : "memory");
}

// ------------------------------------------------------------------ storage types
template <typename T> struct Store;
template <> struct Store<__half> {
  __device__ static float to_f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
  __device__ static uint16_t from_f(float v) { return __half_as_ushort(__float2half_rn(v)); }
  __device__ static float2 pair(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&w));
  }
};
template <> struct Store<__nv_bfloat16> {
  __device__ static float to_f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
  __device__ static uint16_t from_f(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  __device__ static float2 pair(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
};

template <typename T>
__device__ __forceinline__ float dot8(uint4 w, float4 a, float4 b, float acc) {
  float2 f;
  f = Store<T>::pair(w.x); acc = fmaf(f.x, a.x, acc); acc = fmaf(f.y, a.y, acc);
  f = Store<T>::pair(w.y); acc = fmaf(f.x, a.z, acc); acc = fmaf(f.y, a.w, acc);
  f = Store<T>::pair(w.z); acc = fmaf(f.x, b.x, acc); acc = fmaf(f.y, b.y, acc);
  f = Store<T>::pair(w.w); acc = fmaf(f.x, b.z, acc); acc = fmaf(f.y, b.w, acc);
  return acc;
}

// ------------------------------------------------------------------ shared state
struct Misc {
  StageCta sc[ST_COUNT];
  Block blk[kMaxBlocksPerCta];
  float rinv[64];          // per-lane 1/rms of the staged input
  float red_v[kConsumerWarps];
  int32_t red_i[kConsumerWarps];
  volatile int32_t abort;  // a consumer saw a failed wait
  int32_t flag;            // broadcast slot
};

struct Smem {
  uint8_t *ring;
  uint64_t *full, *empty;
  float *vbuf, *part;
  Misc *misc;
};

__device__ __forceinline__ uint32_t *sync_at(const KernelArgs &a, int slot) {
  return a.sync + slot * kSyncStride;
}

__device__ void raise_error(const KernelArgs &a, uint32_t code) {
  atomicCAS(sync_at(a, SY_STATUS), 0u, code);
  atomicExch(sync_at(a, SY_ABORT), 1u);
}

// Bounded wait until *ctr >= target.  False on watchdog expiry or abort.
__device__ bool wait_counter(const KernelArgs &a, const uint32_t *ctr, uint32_t target,
                             uint32_t where) {
  if (ld_acquire(ctr) >= target) return true;
  const uint64_t t0 = globaltimer();
  const uint32_t *abortp = sync_at(a, SY_ABORT);
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire(ctr) >= target) return true;
    if ((it & 15) == 0) {
      if (ld_relaxed(abortp)) return false;
      if (globaltimer() - t0 > a.watchdog_ns) {
        raise_error(a, DE_TIMEOUT_COUNTER | (where << 8));
        return false;
      }
    }
  }
}

// Bounded wait on an mbarrier phase.
__device__ bool wait_mbar(const KernelArgs &a, uint64_t *bar, uint32_t parity, uint32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint32_t *abortp = sync_at(a, SY_ABORT);
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15) == 0) {
      if (ld_relaxed(abortp)) return false;
      if (globaltimer() - t0 > a.watchdog_ns) {
        raise_error(a, code);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ producer
struct Producer {
  const KernelArgs &a;
  Smem s;
  uint32_t T = 0;          // tiles issued
  const uint8_t *cur = nullptr;
  uint64_t policy;
  bool ok = true;

  __device__ Producer(const KernelArgs &a_, Smem s_) : a(a_), s(s_) { policy = policy_evict_first(); }

  __device__ void stage(int k) {
    if (!ok) return;
    const StageShape sh = a.shape[k];
    const StageCta &c = s.misc->sc[k];
    const int NS = a.ring_slots;
    for (int bi = 0; bi < c.nblk; ++bi) {
      const Block b = s.misc->blk[c.blk_begin + bi];
      for (int r0 = 0; r0 < b.nrows; r0 += sh.R) {
        const int rows = min(sh.R, b.nrows - r0);
        const uint32_t bytes = uint32_t(rows) * uint32_t(sh.KT) * 2u;
        for (int sg = 0; sg < sh.nseg; ++sg) {
          const uint32_t slot = T % NS;
          if (T >= (uint32_t)NS) {
            if (!wait_mbar(a, &s.empty[slot], ((T / NS) - 1) & 1, DE_TIMEOUT_EMPTY | (k << 8))) {
              ok = false;
              return;
            }
          }
          mbar_expect_tx(&s.full[slot], bytes);
          bulk_g2s(s.ring + size_t(slot) * kSlotBytes, cur, bytes, &s.full[slot], policy);
          cur += bytes;
          ++T;
        }
      }
    }
  }

  __device__ void run(int cta) {
    const uint8_t *base = a.wstream + a.cta_stream_off[cta];
    const int L = a.n_layers;
    const bool lanes = a.n_lanes > 1;
    for (int step = 0; step < a.n_steps && ok; ++step) {
      const bool lm = a.logits_every_step || step == a.n_steps - 1;
      cur = base;
      for (int l = 0; l < L && ok; ++l) {
        stage(ST_QKV);
        if (lanes && l >= 1) stage(ST_MIX);
        stage(ST_O);
        stage(ST_GU);
        stage(ST_D);
      }
      if (lm) {
        if (lanes) stage(ST_MIX);
        stage(ST_LM);
      }
    }
    // Leave no copy in flight: each slot holds at most one outstanding copy,
    // the most recent one issued into it.
    const uint32_t NS = a.ring_slots;
    const uint32_t first = T > NS ? T - NS : 0;
    for (uint32_t t = first; t < T; ++t) {
      if (!mbar_try_wait(&s.full[t % NS], (t / NS) & 1)) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&s.full[t % NS], (t / NS) & 1)) {
          if (globaltimer() - t0 > a.watchdog_ns) break;
        }
      }
    }
  }
};

// ------------------------------------------------------------------ consumer
template <typename T>
struct Consumer {
  const KernelArgs &a;
  Smem s;
  const int tid, warp, lane, cta;
  uint32_t Tbase = 0;   // tiles consumed before the current stage
  int step = 0, l = 0, tok = 0, p = 0;
  uint32_t lm_count = 0;

  __device__ Consumer(const KernelArgs &a_, Smem s_, int tid_, int cta_)
      : a(a_), s(s_), tid(tid_), warp(tid_ >> 5), lane(tid_ & 31), cta(cta_) {}

  __device__ bool aborted() const { return s.misc->abort != 0; }

  // thread 0 waits for a counter, everyone learns the outcome
  __device__ bool gate(int slot, uint32_t target, uint32_t where) {
    if (tid == 0) {
      if (!wait_counter(a, sync_at(a, slot), target, where)) s.misc->abort = 1;
      __threadfence();
    }
    cbar();
    return !aborted();
  }

  __device__ void signal(int slot) {
    cbar();
    if (tid == 0) {
      __threadfence();
      red_release_add(sync_at(a, slot), 1u);
    }
  }

  // ---- stage inputs
  __device__ float xin(int i) const {
    // residual entering the current layer, plus the delayed sum landing here
    float v = (l == 0) ? Store<T>::to_f(a.embed[size_t(tok) * a.d_model + i]) : __ldcg(a.x + i);
    if (a.n_lanes > 1 && l >= a.lane_delay)
      v += __ldcg(a.dsum + size_t((l - a.lane_delay) % a.lane_delay) * a.d_model + i);
    return v;
  }

  // vbuf = RMSNorm of vbuf (already holding the raw input) with `gain`,
  // per lane slice of width `seg`.
  __device__ void norm_vbuf(const float *gain, int n, int seg) {
    float *v = s.vbuf;
    const int nseg = n / seg;
    cbar();
    if (nseg == 1) {
      float acc = 0.f;
      for (int i = tid; i < n; i += kNC) acc = fmaf(v[i], v[i], acc);
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) s.misc->red_v[warp] = acc;
      cbar();
      if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) t += s.misc->red_v[w];
        s.misc->rinv[0] = rsqrtf(t / float(n) + a.rms_eps);
      }
    } else {
      for (int sgi = warp; sgi < nseg; sgi += kConsumerWarps) {
        float acc = 0.f;
        for (int i = lane; i < seg; i += 32) acc = fmaf(v[sgi * seg + i], v[sgi * seg + i], acc);
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) s.misc->rinv[sgi] = rsqrtf(acc / float(seg) + a.rms_eps);
      }
    }
    cbar();
    for (int i = tid; i < n; i += kNC) v[i] = v[i] * s.misc->rinv[i / seg] * gain[i];
    cbar();
  }

  __device__ void load_vbuf(const float *src, int n) {
    for (int i = tid; i < n; i += kNC) s.vbuf[i] = __ldcg(src + i);
    cbar();
  }

  // ---- GEMV over the stage's tiles: partial sums into s.part
  template <int R>
  __device__ void tile_dot(const uint8_t *tile, const float *vin, int KT, int rows, int nseg,
                           int prow, int sg) {
    const int nch = KT >> 3;
    const uint4 *w4 = reinterpret_cast<const uint4 *>(tile);
    const float4 *v4 = reinterpret_cast<const float4 *>(vin);
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    for (int c = lane; c < nch; c += 32) {
      const float4 va = v4[2 * c], vb = v4[2 * c + 1];
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) acc[r] = dot8<T>(w4[r * nch + c], va, vb, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float v = acc[r];
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) s.part[(prow + r) * nseg + sg] = acc[r];
    }
  }

  __device__ void gemv(int k) {
    const StageShape sh = a.shape[k];
    const StageCta &c = s.misc->sc[k];
    const uint32_t NS = a.ring_slots;
    bool ok = !aborted();
    for (int bi = 0; bi < c.nblk && ok; ++bi) {
      const Block b = s.misc->blk[c.blk_begin + bi];
      const int nrg = (b.nrows + sh.R - 1) / sh.R;
      const int nt = nrg * sh.nseg;
      int first = (warp - (b.tile0 % kConsumerWarps) + kConsumerWarps) % kConsumerWarps;
      for (int tl = first; tl < nt; tl += kConsumerWarps) {
        const int g = tl / sh.nseg, sg = tl - g * sh.nseg;
        const int rows = min(sh.R, b.nrows - g * sh.R);
        const uint32_t Tt = Tbase + b.tile0 + tl;
        const uint32_t slot = Tt % NS;
        bool got = true;
        if (lane == 0) got = wait_mbar(a, &s.full[slot], (Tt / NS) & 1, DE_TIMEOUT_FULL | (k << 8));
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          s.misc->abort = 1;
          ok = false;
          break;
        }
        const uint8_t *tile = s.ring + size_t(slot) * kSlotBytes;
        const float *vin = s.vbuf + b.in_off + sg * sh.KT;
        const int prow = b.lrow0 + g * sh.R;
        switch (sh.R) {
          case 1: tile_dot<1>(tile, vin, sh.KT, rows, sh.nseg, prow, sg); break;
          case 2: tile_dot<2>(tile, vin, sh.KT, rows, sh.nseg, prow, sg); break;
          case 4: tile_dot<4>(tile, vin, sh.KT, rows, sh.nseg, prow, sg); break;
          case 8: tile_dot<8>(tile, vin, sh.KT, rows, sh.nseg, prow, sg); break;
          default: tile_dot<16>(tile, vin, sh.KT, rows, sh.nseg, prow, sg); break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[slot]);
      }
    }
    Tbase += c.ntiles;
    cbar();
  }

  __device__ float rowsum(int i, int nseg) const {
    float v = 0.f;
    for (int sg = 0; sg < nseg; ++sg) v += s.part[i * nseg + sg];
    return v;
  }

  // ---- attention over the cache for one KV head group (split-KV)
  __device__ void attention() {
    const int dh = a.head_dim, half = dh >> 1;
    const int Hkv = a.n_kv_heads, G = a.n_heads / a.n_kv_heads;
    const int g = cta % Hkv;
    const int split = cta / Hkv;
    const int nsplit = (a.n_ctas - 1 - g) / Hkv + 1;
    const int Lctx = p + 1;
    const int j0 = int((int64_t)split * Lctx / nsplit);
    const int j1 = int((int64_t)(split + 1) * Lctx / nsplit);
    const bool writer = (split == nsplit - 1);  // its range holds position p
    float *qs = s.vbuf;              // [G][dh] roped, scaled queries
    float *kcur = qs + G * dh;       // [dh] roped, rounded key of position p
    float *vcur = kcur + dh;         // [dh] rounded value of position p
    float *wst = vcur + dh;          // [W][G][dh + 2] per-warp softmax states
    const float *qkv = a.qkv;
    const float2 *cs = a.rope_cs + size_t(p) * half;
    const size_t cache_row = ((size_t(l) * Hkv + g) * a.max_seq + p) * dh;
    for (int idx = tid; idx < (G + 2) * dh; idx += kNC) {
      const int hh = idx / dh, d = idx - hh * dh;
      const int dd = d < half ? d : d - half;
      const float2 c = cs[dd];
      if (hh < G) {
        const float *q = qkv + size_t(g * G + hh) * dh;
        const float v0 = __ldcg(q + d), v1 = __ldcg(q + (d < half ? d + half : d - half));
        const float r = d < half ? v0 * c.x - v1 * c.y : v0 * c.x + v1 * c.y;
        qs[idx] = r * a.attn_scale;
      } else if (hh == G) {
        const float *k = qkv + size_t(a.n_heads) * dh + size_t(g) * dh;
        const float v0 = __ldcg(k + d), v1 = __ldcg(k + (d < half ? d + half : d - half));
        const float r = d < half ? v0 * c.x - v1 * c.y : v0 * c.x + v1 * c.y;
        const uint16_t b = Store<T>::from_f(r);
        kcur[d] = Store<T>::to_f(b);
        if (writer) a.kcache[cache_row + d] = b;
      } else {
        const float *vv = qkv + size_t(a.n_heads + Hkv) * dh + size_t(g) * dh;
        const uint16_t b = Store<T>::from_f(__ldcg(vv + d));
        vcur[d] = Store<T>::to_f(b);
        if (writer) a.vcache[cache_row + d] = b;
      }
    }
    cbar();
    // each warp folds positions j0 + warp, j0 + warp + W, ... with an online softmax
    const int dpl = dh >> 5;  // dims per lane: 4 (dh 128) or 2 (dh 64)
    float m[4], lsum[4], o[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[i] = -INFINITY;
      lsum[i] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    }
    const uint16_t *kbase = a.kcache + ((size_t(l) * Hkv + g) * a.max_seq) * dh;
    const uint16_t *vbase = a.vcache + ((size_t(l) * Hkv + g) * a.max_seq) * dh;
    for (int j = j0 + warp; j < j1; j += kConsumerWarps) {
      float kv[4], vv[4];
      if (j == p) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < dpl) { kv[e] = kcur[lane * dpl + e]; vv[e] = vcur[lane * dpl + e]; }
      } else if (dpl == 4) {
        const uint2 kw = __ldcg(reinterpret_cast<const uint2 *>(kbase + size_t(j) * dh) + lane);
        const uint2 vw = __ldcg(reinterpret_cast<const uint2 *>(vbase + size_t(j) * dh) + lane);
        float2 f;
        f = Store<T>::pair(kw.x); kv[0] = f.x; kv[1] = f.y;
        f = Store<T>::pair(kw.y); kv[2] = f.x; kv[3] = f.y;
        f = Store<T>::pair(vw.x); vv[0] = f.x; vv[1] = f.y;
        f = Store<T>::pair(vw.y); vv[2] = f.x; vv[3] = f.y;
      } else {
        const uint32_t kw = __ldcg(reinterpret_cast<const unsigned int *>(kbase + size_t(j) * dh) + lane);
        const uint32_t vw = __ldcg(reinterpret_cast<const unsigned int *>(vbase + size_t(j) * dh) + lane);
        float2 f;
        f = Store<T>::pair(kw); kv[0] = f.x; kv[1] = f.y;
        f = Store<T>::pair(vw); vv[0] = f.x; vv[1] = f.y;
        kv[2] = kv[3] = vv[2] = vv[3] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i < G) {
          float sc = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (e < dpl) sc = fmaf(qs[i * dh + lane * dpl + e], kv[e], sc);
          for (int of = 16; of; of >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, of);
          const float mn = fmaxf(m[i], sc);
          const float corr = expf(m[i] - mn);
          const float pj = expf(sc - mn);
          lsum[i] = lsum[i] * corr + pj;
#pragma unroll
          for (int e = 0; e < 4; ++e) o[i][e] = o[i][e] * corr + pj * vv[e];
          m[i] = mn;
        }
      }
    }
    const int st = dh + 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i < G) {
        float *w = wst + (size_t(warp) * G + i) * st;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < dpl) w[lane * dpl + e] = o[i][e];
        if (lane == 0) { w[dh] = m[i]; w[dh + 1] = lsum[i]; }
      }
    }
    cbar();
    // combine the warps into this CTA's partial for each query head
    for (int idx = tid; idx < G * dh; idx += kNC) {
      const int i = idx / dh, d = idx - i * dh;
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, wst[(size_t(w) * G + i) * st + dh]);
      float Ls = 0.f, O = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float *ws = wst + (size_t(w) * G + i) * st;
          const float f = expf(ws[dh] - M);
          Ls += ws[dh + 1] * f;
          O += ws[d] * f;
        }
      }
      float *dst = a.attn_part + (size_t(g * G + i) * a.max_split + split) * st;
      dst[d] = O;
      if (d == 0) { dst[dh] = M; dst[dh + 1] = Ls; }
    }
    cbar();
    const uint32_t epoch = uint32_t(step) * a.n_layers + l + 1;
    if (tid == 0) {
      __threadfence();
      const uint32_t old = atom_acq_rel_add(sync_at(a, SY_ATTN0 + g), 1u);
      s.misc->flag = (old + 1 == epoch * uint32_t(nsplit)) ? 1 : 0;
      __threadfence();
    }
    cbar();
    if (s.misc->flag) {
      // last split of this group: merge all splits into attn_o
      for (int idx = tid; idx < G * dh; idx += kNC) {
        const int i = idx / dh, d = idx - i * dh;
        const float *src = a.attn_part + size_t(g * G + i) * a.max_split * st;
        float M = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, __ldcg(src + size_t(sp) * st + dh));
        float Ls = 0.f, O = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) {
          const float *ps = src + size_t(sp) * st;
          const float f = expf(__ldcg(ps + dh) - M);
          Ls += __ldcg(ps + dh + 1) * f;
          O += __ldcg(ps + d) * f;
        }
        a.attn_o[size_t(g * G + i) * dh + d] = O / Ls;
      }
      signal(SY_OREADY);
    }
  }

  // ---- LM head epilogue: logits and the CTA's share of the argmax
  __device__ void lm_epilogue() {
    const StageCta &c = s.misc->sc[ST_LM];
    const int nseg = a.shape[ST_LM].nseg;
    float best = -INFINITY;
    int bidx = 0x7fffffff;
    for (int i = tid; i < c.nout; i += kNC) {
      const float v = rowsum(i, nseg);
      const int row = c.row0 + i;
      if (a.logits_out) a.logits_out[size_t(step) * a.vocab + row] = v;
      if (v > best || (v == best && row < bidx)) { best = v; bidx = row; }
    }
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
      if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
    }
    if (lane == 0) { s.misc->red_v[warp] = best; s.misc->red_i[warp] = bidx; }
    cbar();
    if (tid == 0 && c.nout > 0) {
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float ov = s.misc->red_v[w];
        const int oi = s.misc->red_i[w];
        if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
      }
      const uint32_t fb = __float_as_uint(best);
      const uint32_t ord = (fb & 0x80000000u) ? ~fb : (fb | 0x80000000u);
      const unsigned long long key =
          (static_cast<unsigned long long>(ord) << 32) | (0xffffffffu - uint32_t(bidx));
      atomicMax(a.keys + step, key);
    }
  }

  __device__ void run() {
    const int L = a.n_layers, d = a.d_model;
    const bool lanes = a.n_lanes > 1;
    const int delta = a.lane_delay;
    const uint32_t nc = a.n_ctas;
    tok = a.forced ? a.forced[0] : a.first_token;
    for (step = 0; step < a.n_steps; ++step) {
      p = a.pos0 + step;
      const bool lm = a.logits_every_step || step == a.n_steps - 1;
      for (l = 0; l < L; ++l) {
        const uint32_t e = uint32_t(step) * L + l + 1;  // epoch of this (step, layer)
        // ---------------- RMSNorm + QKV
        if (l > 0 && !gate(SY_X2, (e - 1) * nc, 0x10 + ST_QKV)) goto done;
        for (int i = tid; i < d; i += kNC) s.vbuf[i] = xin(i);
        norm_vbuf(a.gain_attn + size_t(l) * d, d, a.lane_width);
        gemv(ST_QKV);
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_QKV];
          const int nseg = a.shape[ST_QKV].nseg;
          for (int i = tid; i < c.nout; i += kNC) a.qkv[c.row0 + i] = rowsum(i, nseg);
        }
        if (!(a.skip_signal_cta == cta && step == 0 && l == 0)) signal(SY_QKV);
        // ---------------- delayed cross-lane sum of the previous layer
        if (lanes && l >= 1) {
          load_vbuf(a.ubuf + size_t((l - 1) & 1) * d, d);
          gemv(ST_MIX);
          if (aborted()) goto done;
          const StageCta &c = s.misc->sc[ST_MIX];
          const int nseg = a.shape[ST_MIX].nseg;
          float *dst = a.dsum + size_t((l - 1) % delta) * d;
          for (int i = tid; i < c.nout; i += kNC) dst[c.row0 + i] = rowsum(i, nseg);
        }
        // ---------------- attention
        if (!gate(SY_QKV, e * nc, 0x20)) goto done;
        attention();
        // ---------------- O + residual
        if (!gate(SY_OREADY, e * uint32_t(a.n_kv_heads), 0x30)) goto done;
        load_vbuf(a.attn_o, a.n_heads * a.head_dim);
        gemv(ST_O);
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_O];
          const int nseg = a.shape[ST_O].nseg;
          for (int i = tid; i < c.nout; i += kNC) {
            const int r = c.row0 + i;
            const float v = rowsum(i, nseg);
            a.x[r] = xin(r) + v;
            if (lanes) a.ubuf[size_t(l & 1) * d + r] = v;
          }
        }
        signal(SY_X1);
        // ---------------- RMSNorm + gate/up + SwiGLU
        if (!gate(SY_X1, e * nc, 0x40)) goto done;
        for (int i = tid; i < d; i += kNC) s.vbuf[i] = __ldcg(a.x + i);
        norm_vbuf(a.gain_ffn + size_t(l) * d, d, a.lane_width);
        gemv(ST_GU);
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_GU];
          const int nseg = a.shape[ST_GU].nseg;
          for (int i = tid; i < c.nout; i += kNC) {
            const float gt = rowsum(i, nseg), up = rowsum(c.nout + i, nseg);
            a.hbuf[c.row0 + i] = gt / (1.f + expf(-gt)) * up;
          }
        }
        signal(SY_H);
        // ---------------- down + residual
        if (!gate(SY_H, e * nc, 0x50)) goto done;
        load_vbuf(a.hbuf, a.ffn_dim);
        gemv(ST_D);
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_D];
          const int nseg = a.shape[ST_D].nseg;
          for (int i = tid; i < c.nout; i += kNC) {
            const int r = c.row0 + i;
            const float v = rowsum(i, nseg);
            a.x[r] = __ldcg(a.x + r) + v;
            if (lanes) {
              float *u = a.ubuf + size_t(l & 1) * d + r;
              *u = __ldcg(u) + v;
            }
          }
        }
        signal(SY_X2);
      }
      if (lm) {
        ++lm_count;
        if (!gate(SY_X2, (uint32_t(step) * L + L) * nc, 0x60)) goto done;
        if (lanes) {
          // the last layer's delayed sum, flushed before the final norm
          load_vbuf(a.ubuf + size_t((L - 1) & 1) * d, d);
          gemv(ST_MIX);
          if (aborted()) goto done;
          const StageCta &c = s.misc->sc[ST_MIX];
          const int nseg = a.shape[ST_MIX].nseg;
          float *dst = a.dsum + size_t((L - 1) % delta) * d;
          for (int i = tid; i < c.nout; i += kNC) dst[c.row0 + i] = rowsum(i, nseg);
          signal(SY_MIXF);
          if (!gate(SY_MIXF, lm_count * nc, 0x70)) goto done;
        }
        for (int i = tid; i < d; i += kNC) {
          float v = __ldcg(a.x + i);
          if (lanes)
            for (int li = (L > delta ? L - delta : 0); li < L; ++li)
              v += __ldcg(a.dsum + size_t(li % delta) * d + i);
          s.vbuf[i] = v;
        }
        norm_vbuf(a.gain_final, d, d);
        gemv(ST_LM);
        if (aborted()) goto done;
        lm_epilogue();
        signal(SY_TOK);
        if (!gate(SY_TOK, lm_count * nc, 0x80)) goto done;
        const unsigned long long key = __ldcg(a.keys + step);
        const int next = int(0xffffffffu - uint32_t(key & 0xffffffffull));
        if (cta == 0 && tid == 0) a.out_tokens[step] = next;
        tok = next;
      }
      if (a.forced && step + 1 < a.n_steps) tok = a.forced[step + 1];
    }
  done:
    return;
  }
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) monokernel(const KernelArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int tid = threadIdx.x;
  const int cta = blockIdx.x;
  const int NS = a.ring_slots;
  Smem s;
  s.ring = smem_raw;
  s.full = reinterpret_cast<uint64_t *>(smem_raw + size_t(NS) * kSlotBytes);
  s.empty = s.full + NS;
  s.vbuf = reinterpret_cast<float *>(s.empty + NS);
  s.part = s.vbuf + a.vbuf_floats;
  s.misc = reinterpret_cast<Misc *>(s.part + a.part_floats);

  const int b0 = a.cta_blk_begin[cta], b1 = a.cta_blk_begin[cta + 1];
  for (int i = tid; i < b1 - b0; i += kThreads) s.misc->blk[i] = a.blocks[b0 + i];
  if (tid < ST_COUNT) s.misc->sc[tid] = a.stage_cta[tid * a.n_ctas + cta];
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    s.misc->abort = 0;
    s.misc->flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (tid >= kNC) {
    if (tid == kNC) {
      Producer pr(a, s);
      pr.run(cta);
    }
    __syncwarp();
  } else {
    Consumer<T> c(a, s, tid, cta);
    c.run();
    // a consumer that gave up makes sure the producer stops too
    if (tid == 0 && c.aborted()) atomicExch(sync_at(a, SY_ABORT), 1u);
  }
  __syncthreads();
}

// ------------------------------------------------------------------ weight repack
// Copies each block of canonical row-major rows into tile order: row groups of
// R rows, each split into K/KT column segments stored as R x KT row-major.
__global__ void repack_kernel(const uint16_t *__restrict__ src, uint8_t *__restrict__ dst,
                              const RepackJob *__restrict__ jobs, int njobs) {
  for (int j = blockIdx.x; j < njobs; j += gridDim.x) {
    const RepackJob job = jobs[j];
    const int64_t K = job.K, KT = job.KT, R = job.R;
    const int64_t nvec = int64_t(job.nrows) * K / 8;
    uint16_t *out = reinterpret_cast<uint16_t *>(dst + job.dst_byte);
    for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
      const int64_t e = v * 8;             // element index in row-major source order
      const int64_t i = e / K, k = e - i * K;
      const int64_t g = i / R, ii = i - g * R;
      const int64_t rg = min(R, int64_t(job.nrows) - g * R);
      const int64_t sg = k / KT, kk = k - sg * KT;
      const int64_t o = g * R * K + sg * rg * KT + ii * KT + kk;
      *reinterpret_cast<uint4 *>(out + o) =
          *reinterpret_cast<const uint4 *>(src + job.src_elem + e);
    }
  }
}

// ------------------------------------------------------------------ host entry points
size_t monokernel_smem_bytes(int ring_slots, int vbuf_floats, int part_floats) {
  return size_t(ring_slots) * kSlotBytes + size_t(ring_slots) * 16 +
         size_t(vbuf_floats + part_floats) * 4 + sizeof(Misc);
}

int monokernel_threads() { return kThreads; }

const void *monokernel_fn(int dtype) {
  return dtype == 0 ? reinterpret_cast<const void *>(&monokernel<__half>)
                    : reinterpret_cast<const void *>(&monokernel<__nv_bfloat16>);
}

cudaError_t launch_repack(const uint16_t *src, uint8_t *dst, const RepackJob *jobs, int njobs,
                          cudaStream_t st) {
  if (njobs == 0) return cudaSuccess;
  repack_kernel<<<min(njobs, 4096), 256, 0, st>>>(src, dst, jobs, njobs);
  return cudaGetLastError();
}

}  // namespace kie
