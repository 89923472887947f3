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
// primitive.  Every spin is bounded by an SM-clock watchdog; on expiry
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
static_assert(kNC * 4 == 2048, "staging indexes warp partial sums by element / 2048");

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
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
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

// ------------------------------------------------------------------ profiling build
// With -DKIE_PROFILE every SM accumulates SM-clock cycles per activity and
// writes them to KernelArgs::prof[cta * kProfSlots + slot] at exit.
#ifdef KIE_PROFILE
#define KP_BEGIN(var) long long var = (tid == 0) ? clock64() : 0ll
#define KP_END(var, slot) \
  do { if (tid == 0) s.misc->prof[slot] += clock64() - var; } while (0)
#else
#define KP_BEGIN(var) do {} while (0)
#define KP_END(var, slot) do {} while (0)
#endif

// ------------------------------------------------------------------ shared state
// Position of the next weight tile to issue (thread 0's copy pump).
struct PumpState {
  const uint8_t *cur;        // next byte of this CTA's weight stream
  uint32_t T;                // tiles issued
  int32_t step, l, si, bi, r0, nseq;
  int32_t seq[6];            // stage kinds of the current layer (or tail)
  int32_t done;
};

struct Misc {
  StageCta sc[ST_COUNT];
  Block blk[kMaxBlocksPerCta];
  float red_sq[4 * kConsumerWarps];  // per-warp sums of squares while staging
  float red_v[kConsumerWarps];
  int32_t red_i[kConsumerWarps];
  volatile int32_t abort;  // a consumer saw a failed wait
  int32_t flag;            // broadcast slot
  long long prof[kProfSlots];
  PumpState pump;   // next tile to copy into the ring
  PumpState pf;     // next tile to prefetch into L2 (runs ahead of `pump`)
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

// Watchdog arithmetic uses the SM cycle counter (cheap to read); the limit in
// cycles assumes at most 2 GHz, so a wait gives up after at least watchdog_ns.
// The shared abort flag (a global load, about a microsecond) is polled only
// every ~64K cycles so that it never delays noticing a completed wait.
constexpr long long kAbortPollCycles = 1 << 16;

// Bounded wait until *ctr >= target.  False on watchdog expiry or abort.
template <typename PumpT>
__device__ bool wait_counter(const KernelArgs &a, const uint32_t *ctr, uint32_t target,
                             uint32_t where, PumpT &&pump) {
  if (ld_acquire(ctr) >= target) return true;
  const long long t0 = clock64(), limit = (long long)a.watchdog_ns * 2;
  long long next_poll = kAbortPollCycles;
  const uint32_t *abortp = sync_at(a, SY_ABORT);
  for (;;) {
    if (ld_acquire(ctr) >= target) return true;
    pump();
    const long long el = clock64() - t0;
    if (el > next_poll) {
      next_poll = el + kAbortPollCycles;
      if (ld_relaxed(abortp)) return false;
      if (el > limit) {
        raise_error(a, DE_TIMEOUT_COUNTER | (where << 8));
        return false;
      }
    }
  }
}

// Bounded wait on an mbarrier phase.
template <typename PumpT>
__device__ bool wait_mbar(const KernelArgs &a, uint64_t *bar, uint32_t parity, uint32_t code,
                          PumpT &&pump) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64(), limit = (long long)a.watchdog_ns * 2;
  long long next_poll = kAbortPollCycles;
  const uint32_t *abortp = sync_at(a, SY_ABORT);
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    pump();
    const long long el = clock64() - t0;
    if (el > next_poll) {
      next_poll = el + kAbortPollCycles;
      if (ld_relaxed(abortp)) return false;
      if (el > limit) {
        raise_error(a, code);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ weight pump
// Thread 0 of each CTA issues the CTA's weight tiles, in the order they are
// consumed, into free ring slots: one cp.async.bulk (1-D bulk copy, no tensor
// map, no multicast, L2 evict-first) per tile, completing on the slot's full
// mbarrier.  It never blocks: pump() returns when the next slot is still in
// use, and thread 0 calls it from every wait loop it runs (dependency gates,
// tile waits) and after every tile, so the weight stream keeps flowing while
// the CTA waits for other SMs -- weights do not depend on activations.
struct Pump {
  const KernelArgs &a;
  Smem s;
  __device__ Pump(const KernelArgs &a_, Smem s_) : a(a_), s(s_) {}

  __device__ bool lm_step(int step) const { return a.logits_every_step || step == a.n_steps - 1; }

  __device__ void load_seq(PumpState &p) const {
    p.nseq = 0;
    const bool lanes = a.n_lanes > 1;
    if (p.l < a.n_layers) {
      p.seq[p.nseq++] = ST_QKV;
      if (lanes && p.l >= 1) p.seq[p.nseq++] = ST_MIX;
      p.seq[p.nseq++] = ST_O;
      p.seq[p.nseq++] = ST_GU;
      p.seq[p.nseq++] = ST_D;
    } else if (lm_step(p.step)) {
      if (lanes) p.seq[p.nseq++] = ST_MIX;
      p.seq[p.nseq++] = ST_LM;
    }
  }

  // move (si, bi, r0) forward to the next tile that exists
  __device__ void normalize(PumpState &p, const uint8_t *base) const {
    while (!p.done) {
      if (p.si < p.nseq) {
        const StageCta &c = s.misc->sc[p.seq[p.si]];
        if (p.bi < c.nblk) {
          if (p.r0 < s.misc->blk[c.blk_begin + p.bi].nrows) return;
          ++p.bi;
          p.r0 = 0;
          continue;
        }
        ++p.si;
        p.bi = 0;
        p.r0 = 0;
        continue;
      }
      p.si = p.bi = p.r0 = 0;
      if (p.l < a.n_layers) {
        ++p.l;
      } else {
        ++p.step;
        p.l = 0;
        p.cur = base;
        if (p.step >= a.n_steps) {
          p.done = 1;
          return;
        }
      }
      load_seq(p);
    }
  }

  __device__ void init_state(PumpState &p, int cta) const {
    p.cur = a.wstream + a.cta_stream_off[cta];
    p.T = 0;
    p.step = p.l = p.si = p.bi = p.r0 = 0;
    p.done = a.n_steps > 0 ? 0 : 1;
    load_seq(p);
    normalize(p, p.cur);
  }

  __device__ uint32_t tile_bytes(const PumpState &p) const {
    const int k = p.seq[p.si];
    const StageShape &sh = a.shape[k];
    const Block &b = s.misc->blk[s.misc->sc[k].blk_begin + p.bi];
    return uint32_t(min(sh.R, b.nrows - p.r0)) * uint32_t(sh.K) * 2u;
  }

  __device__ void advance(PumpState &p, uint32_t bytes, const uint8_t *base) const {
    p.cur += bytes;
    ++p.T;
    p.r0 += a.shape[p.seq[p.si]].R;
    normalize(p, base);
  }

  __device__ void init(int cta) {
    init_state(s.misc->pump, cta);
    init_state(s.misc->pf, cta);
  }

  // Copy tiles into every free ring slot; returns when the next slot is busy.
  __device__ void pump(int cta) {
    PumpState &p = s.misc->pump;
    const uint32_t NS = a.ring_slots;
    const uint8_t *base = a.wstream + a.cta_stream_off[cta];
    while (!p.done) {
      const uint32_t slot = p.T % NS;
      if (p.T >= NS && !mbar_try_wait(&s.empty[slot], ((p.T / NS) - 1) & 1)) return;
      const uint32_t bytes = tile_bytes(p);
      mbar_expect_tx(&s.full[slot], bytes);
      bulk_g2s(s.ring + size_t(slot) * kSlotBytes, p.cur, bytes, &s.full[slot], policy_evict_first());
      advance(p, bytes, base);
    }
  }

  // While the ring is full, pull the next l2_prefetch_tiles tiles into L2 so
  // that HBM keeps streaming and the ring refills from L2 once slots free up.
  __device__ void prefetch(int cta) {
    PumpState &q = s.misc->pf;
    const uint32_t T = s.misc->pump.T;
    const uint8_t *base = a.wstream + a.cta_stream_off[cta];
    while (!q.done && q.T < T + uint32_t(a.l2_prefetch_tiles)) {
      const uint32_t bytes = tile_bytes(q);
      if (q.T >= T) prefetch_l2(q.cur, bytes);
      advance(q, bytes, base);
    }
  }

  // The producer warp's loop: fill free slots, prefetch ahead into L2, then
  // sleep on the next slot's empty barrier until every consumer warp released
  // it (bounded by the watchdog).
  __device__ void run(int cta) {
    init(cta);
    PumpState &p = s.misc->pump;
    const uint32_t NS = a.ring_slots;
    while (!p.done) {
      pump(cta);
      if (p.done) break;
      prefetch(cta);
      const uint32_t slot = p.T % NS;
#ifdef KIE_PROFILE
      const long long tw = clock64();
#endif
      if (!wait_mbar(a, &s.empty[slot], ((p.T / NS) - 1) & 1, DE_TIMEOUT_EMPTY, [] {})) break;
#ifdef KIE_PROFILE
      s.misc->prof[PF_PROD_EMPTY] += clock64() - tw;
#endif
    }
    drain();
  }

  // Before the CTA exits: each slot holds at most one outstanding copy, the
  // last one issued into it; wait (bounded) until those have landed.
  __device__ void drain() {
    const uint32_t NS = a.ring_slots, T = s.misc->pump.T;
    const uint32_t first = T > NS ? T - NS : 0;
    for (uint32_t t = first; t < T; ++t) {
      if (!mbar_try_wait(&s.full[t % NS], (t / NS) & 1)) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&s.full[t % NS], (t / NS) & 1)) {
          if (clock64() - t0 > (long long)a.watchdog_ns * 2) break;
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
  uint32_t slot = 0, phase = 0;   // ring position of the next tile (every warp sees every tile)
  int step = 0, l = 0, tok = 0, p = 0;
  uint32_t lm_count = 0;

  __device__ Consumer(const KernelArgs &a_, Smem s_, int tid_, int cta_)
      : a(a_), s(s_), tid(tid_), warp(tid_ >> 5), lane(tid_ & 31), cta(cta_) {}

  __device__ bool aborted() const { return s.misc->abort != 0; }

  // thread 0 waits for a counter, everyone learns the outcome
  __device__ bool gate(int slot, uint32_t target, uint32_t where) {
    if (tid == 0) {
#ifdef KIE_PROFILE
      const long long t0 = clock64();
#endif
      if (!wait_counter(a, sync_at(a, slot), target, where, [] {})) s.misc->abort = 1;
#ifdef KIE_PROFILE
      s.misc->prof[PF_GATE] += clock64() - t0;
      s.misc->prof[PF_GATE_K + slot] += clock64() - t0;
      s.misc->prof[PF_NGATE] += 1;
#endif
    }
    cbar();
    return !aborted();
  }

  __device__ void signal(int slot) {
    KP_BEGIN(t_sig);
    cbar();
    if (tid == 0) red_release_add(sync_at(a, slot), 1u);
    KP_END(t_sig, PF_SIGNAL);
  }

  // ---- stage inputs
  __device__ float xin(int i) const {
    // residual entering the current layer, plus the delayed sum landing here
    float v = (l == 0) ? Store<T>::to_f(a.embed[size_t(tok) * a.d_model + i]) : __ldcg(a.x + i);
    if (a.n_lanes > 1 && l >= a.lane_delay)
      v += __ldcg(a.dsum + size_t((l - a.lane_delay) % a.lane_delay) * a.d_model + i);
    return v;
  }

  // elements 4j..4j+3 of the residual entering the current layer
  __device__ float4 xin4(int j) const {
    float4 v;
    if (l == 0) {
      const uint2 w = *reinterpret_cast<const uint2 *>(a.embed + size_t(tok) * a.d_model + 4 * j);
      const float2 lo = Store<T>::pair(w.x), hi = Store<T>::pair(w.y);
      v = make_float4(lo.x, lo.y, hi.x, hi.y);
    } else {
      v = __ldcg(reinterpret_cast<const float4 *>(a.x) + j);
    }
    if (a.n_lanes > 1 && l >= a.lane_delay) {
      const float4 q = __ldcg(reinterpret_cast<const float4 *>(
                                  a.dsum + size_t((l - a.lane_delay) % a.lane_delay) * a.d_model) + j);
      v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
    }
    return v;
  }

  // vbuf[0..n) = RMSNorm(src) * gain, per lane slice of width seg (a
  // multiple of 128).  src(i4) returns elements 4*i4 .. 4*i4+3.  Each thread
  // holds up to 4 float4 groups; warp partial sums of squares go through
  // shared memory and every thread adds up the ones of its own slice.
  template <typename Src>
  __device__ void stage_norm(Src src, const float *gain, int n, int seg) {
    KP_BEGIN(t_norm);
    const int ng = n >> 2;
    float4 *vb = reinterpret_cast<float4 *>(s.vbuf);
    float4 *gb = vb + ng;   // the gains, staged beside the input
    for (int q = 0; q * kNC < ng; ++q) {
      const int j = tid + q * kNC;
      float ss = 0.f;
      if (j < ng) {
        const float4 v = src(j);
        gb[j] = *reinterpret_cast<const float4 *>(gain + 4 * j);
        vb[j] = v;
        ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s.misc->red_sq[q * kConsumerWarps + warp] = ss;
    }
    cbar();
    for (int q = 0; q * kNC < ng; ++q) {
      const int j = tid + q * kNC;
      if (j < ng) {
        // the slice holding element 4j covers warps' 128-element ranges
        // e = e0, e0 + 128, ...; range e was summed into red_sq[e / 2048 * 16 + e % 2048 / 128]
        const int e0 = (4 * j) / seg * seg;
        float tot = 0.f;
        for (int e = e0; e < e0 + seg; e += 128) tot += s.misc->red_sq[(e >> 11) * kConsumerWarps + ((e >> 7) & 15)];
        const float r = rsqrtf(tot / float(seg) + a.rms_eps);
        const float4 g = gb[j];
        const float4 v = vb[j];
        vb[j] = make_float4(v.x * r * g.x, v.y * r * g.y, v.z * r * g.z, v.w * r * g.w);
      }
    }
    cbar();
    KP_END(t_norm, PF_STAGE);
  }

  // ---- GEMV over the stage's tiles: partial sums into s.part
  // Every consumer warp waits on every tile in order and handles its row group
  // and column split; its slice of the input vector stays in registers for
  // the whole block.  `vin` is the stage input (shared or global memory).
  __device__ void gemv(int k, const float *vin, bool vin_global) {
    if (a.shape[k].rpw > 1) gemv_impl<true>(k, vin, vin_global);
    else gemv_impl<false>(k, vin, vin_global);
  }

  template <bool MULTI>
  __device__ void gemv_impl(int k, const float *vin, bool vin_global) {
    KP_BEGIN(t_gemv);
    const StageShape sh = a.shape[k];
    const StageCta &c = s.misc->sc[k];
    const int rg = warp / sh.nseg, split = warp - rg * sh.nseg;
    const int row0 = rg * sh.rpw;               // first row of this warp inside a tile
    const bool active = row0 < sh.R;
    const int nchunk = sh.rpw * sh.cps;         // chunks this warp covers per tile (<= 128)
    // Per-lane chunk layout, the same for every tile of the stage: byte offset
    // inside the tile, row inside the tile (INT_MAX if unused), input column.
    uint32_t off[4];
    int crow[4], ccol[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ci = lane + 32 * i;
      const int rr = ci / sh.cps, cc = ci - rr * sh.cps;
      const bool valid = active && ci < nchunk;
      crow[i] = valid ? row0 + rr : 0x7fffffff;
      ccol[i] = (split * sh.cps + cc) * 8;
      off[i] = uint32_t((row0 + rr) * sh.K + ccol[i]) * 2u;
    }
    bool ok = !aborted();
    for (int bi = 0; bi < c.nblk && ok; ++bi) {
      const Block b = s.misc->blk[c.blk_begin + bi];
      // this warp's slice of the input vector, kept in registers for the block
      float vr[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (crow[i] != 0x7fffffff) {
          const float *src = vin + b.in_off + ccol[i];
          float4 x0, x1;
          if (vin_global) { x0 = __ldcg(reinterpret_cast<const float4 *>(src)); x1 = __ldcg(reinterpret_cast<const float4 *>(src) + 1); }
          else { x0 = reinterpret_cast<const float4 *>(src)[0]; x1 = reinterpret_cast<const float4 *>(src)[1]; }
          vr[i][0] = x0.x; vr[i][1] = x0.y; vr[i][2] = x0.z; vr[i][3] = x0.w;
          vr[i][4] = x1.x; vr[i][5] = x1.y; vr[i][6] = x1.z; vr[i][7] = x1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) vr[i][e] = 0.f;
        }
      }
      // Tiles go in batches of `batch` (4 / rpw) tiles: each tile's dot
      // products are folded into one value per (tile, row) and its slot is
      // released at once; the batch's 4 values are then reduced across the
      // warp together (transposed butterfly: 6 shuffles for 4 values).
      const int ntile = (b.nrows + sh.R - 1) / sh.R;
      const int batch = MULTI ? 4 / sh.rpw : 4;
      for (int t0 = 0; t0 < ntile && ok; t0 += batch) {
        float val[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int bt = 0; bt < 4; ++bt) {
          if (bt < batch && t0 + bt < ntile) {
            bool got = true;
#ifdef KIE_PROFILE
            const long long tw = (tid == 0) ? clock64() : 0ll;
#endif
            if (lane == 0) got = wait_mbar(a, &s.full[slot], phase, DE_TIMEOUT_FULL | (k << 8), [] {});
#ifdef KIE_PROFILE
            if (tid == 0) s.misc->prof[PF_FULLWAIT] += clock64() - tw;
#endif
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got) {
              s.misc->abort = 1;
              ok = false;
            } else {
              const int rows = min(sh.R, b.nrows - (t0 + bt) * sh.R);
              const uint8_t *tile = s.ring + size_t(slot) * kSlotBytes;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if (crow[i] < rows) {
                  const float4 va = make_float4(vr[i][0], vr[i][1], vr[i][2], vr[i][3]);
                  const float4 vb = make_float4(vr[i][4], vr[i][5], vr[i][6], vr[i][7]);
                  const float d = dot8<T>(*reinterpret_cast<const uint4 *>(tile + off[i]), va, vb, 0.f);
                  // value index: tile bt of the batch, row crow[i] - row0 of the
                  // warp's rows (uniform across lanes); < 4 because batch * rpw == 4
                  if (!MULTI) {
                    val[bt] += d;
                  } else {
                    const int vidx = bt * sh.rpw + (crow[i] - row0);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                      if (j == vidx) val[j] += d;
                  }
                }
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(&s.empty[slot]);
              if (++slot == uint32_t(a.ring_slots)) { slot = 0; phase ^= 1u; }
            }
          }
        }
        if (!ok) break;
        // transposed butterfly: after it, lane l holds the warp sum of value (l >> 3) & 3
        const bool b4 = lane & 16, b3 = lane & 8;
        const float r0 = __shfl_xor_sync(0xffffffffu, b4 ? val[0] : val[2], 16);
        const float r1 = __shfl_xor_sync(0xffffffffu, b4 ? val[1] : val[3], 16);
        const float k0 = (b4 ? val[2] : val[0]) + r0;
        const float k1 = (b4 ? val[3] : val[1]) + r1;
        const float r2 = __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
        float v = (b3 ? k1 : k0) + r2;
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if (active && (lane & 7) == 0) {
          const int vi = lane >> 3;                        // value index 0..3
          const int bt = MULTI ? vi / sh.rpw : vi;          // tile within the batch
          const int r = MULTI ? vi - bt * sh.rpw : 0;       // row within the warp's rows
          const int t = t0 + bt;
          if (t < ntile && r < sh.rpw) {
            const int rows = min(sh.R, b.nrows - t * sh.R);
            if (row0 + r < rows) s.part[(b.lrow0 + t * sh.R + row0 + r) * sh.nseg + split] = v;
          }
        }
      }
    }
    Tbase += c.ntiles;
    cbar();
    KP_END(t_gemv, k == ST_LM ? PF_LM : PF_GEMV);
    KP_END(t_gemv, PF_GEMV_K + k);
  }

  __device__ float rowsum(int i, int nseg) const {
    float v = 0.f;
    for (int sg = 0; sg < nseg; ++sg) v += s.part[i * nseg + sg];
    return v;
  }

  // ---- attention over the cache for one KV head group (split-KV)
  __device__ void attention() {
    KP_BEGIN(t_attn);
    attention_body();
    KP_END(t_attn, PF_ATTN);
  }

  __device__ void attention_body() {
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
      const uint32_t old = atom_acq_rel_add(sync_at(a, SY_ATTN0 + g), 1u);
      s.misc->flag = (old + 1 == epoch * uint32_t(nsplit)) ? 1 : 0;
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
    KP_BEGIN(t_total);
    run_body();
    KP_END(t_total, PF_TOTAL);
  }

  __device__ void run_body() {
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
        stage_norm([=](int j) { return xin4(j); }, a.gain_attn + size_t(l) * d, d, a.lane_width);
        gemv(ST_QKV, s.vbuf, false);
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_QKV];
          const int nseg = a.shape[ST_QKV].nseg;
          for (int i = tid; i < c.nout; i += kNC) a.qkv[c.row0 + i] = rowsum(i, nseg);
        }
        if (!(a.skip_signal_cta == cta && step == 0 && l == 0)) signal(SY_QKV);
        // ---------------- delayed cross-lane sum of the previous layer
        if (lanes && l >= 1) {
          gemv(ST_MIX, a.ubuf + size_t((l - 1) & 1) * d, true);
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
        {
          // residual rows this CTA updates, fetched while the GEMV runs
          const StageCta &c = s.misc->sc[ST_O];
          const float xr = tid < c.nout ? xin(c.row0 + tid) : 0.f;
          gemv(ST_O, a.attn_o, true);
          if (aborted()) goto done;
          const int nseg = a.shape[ST_O].nseg;
          if (tid < c.nout) {
            const int r = c.row0 + tid;
            const float v = rowsum(tid, nseg);
            a.x[r] = xr + v;
            if (lanes) a.ubuf[size_t(l & 1) * d + r] = v;
          }
          for (int i = tid + kNC; i < c.nout; i += kNC) {
            const int r = c.row0 + i;
            const float v = rowsum(i, nseg);
            a.x[r] = xin(r) + v;
            if (lanes) a.ubuf[size_t(l & 1) * d + r] = v;
          }
        }
        signal(SY_X1);
        // ---------------- RMSNorm + gate/up + SwiGLU
        if (!gate(SY_X1, e * nc, 0x40)) goto done;
        stage_norm([=](int j) { return __ldcg(reinterpret_cast<const float4 *>(a.x) + j); },
                   a.gain_ffn + size_t(l) * d, d, a.lane_width);
        gemv(ST_GU, s.vbuf, false);
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
        {
          const StageCta &c = s.misc->sc[ST_D];
          const float xr = tid < c.nout ? __ldcg(a.x + c.row0 + tid) : 0.f;
          gemv(ST_D, a.hbuf, true);
          if (aborted()) goto done;
          const int nseg = a.shape[ST_D].nseg;
          if (tid < c.nout && !lanes) a.x[c.row0 + tid] = xr + rowsum(tid, nseg);
          for (int i = (lanes ? tid : tid + kNC); i < c.nout; i += kNC) {
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
          gemv(ST_MIX, a.ubuf + size_t((L - 1) & 1) * d, true);
          if (aborted()) goto done;
          const StageCta &c = s.misc->sc[ST_MIX];
          const int nseg = a.shape[ST_MIX].nseg;
          float *dst = a.dsum + size_t((L - 1) % delta) * d;
          for (int i = tid; i < c.nout; i += kNC) dst[c.row0 + i] = rowsum(i, nseg);
          signal(SY_MIXF);
          if (!gate(SY_MIXF, lm_count * nc, 0x70)) goto done;
        }
        stage_norm(
            [=](int j) {
              float4 v = __ldcg(reinterpret_cast<const float4 *>(a.x) + j);
              if (lanes)
                for (int li = (L > delta ? L - delta : 0); li < L; ++li) {
                  const float4 q = __ldcg(reinterpret_cast<const float4 *>(a.dsum + size_t(li % delta) * d) + j);
                  v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
                }
              return v;
            },
            a.gain_final, d, d);
        gemv(ST_LM, s.vbuf, false);
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
      mbar_init(&s.empty[i], kConsumerWarps);
    }
    s.misc->abort = 0;
    s.misc->flag = 0;
    for (int i = 0; i < kProfSlots; ++i) s.misc->prof[i] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (tid >= kNC) {
    if (tid == kNC) {
#ifdef KIE_PROFILE
      const long long t0 = clock64();
#endif
      Pump pm(a, s);
      pm.run(cta);
#ifdef KIE_PROFILE
      s.misc->prof[PF_PROD_TOTAL] += clock64() - t0;
      s.misc->prof[PF_TILES] = s.misc->pump.T;
#endif
    }
    __syncwarp();
  } else {
    Consumer<T> c(a, s, tid, cta);
    c.run();
    // a CTA that gave up makes every other CTA (and its own producer) leave
    if (tid == 0 && c.aborted()) atomicExch(sync_at(a, SY_ABORT), 1u);
  }
  __syncthreads();
#ifdef KIE_PROFILE
  if (a.prof && tid < kProfSlots) a.prof[size_t(cta) * kProfSlots + tid] = s.misc->prof[tid];
#endif
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

bool monokernel_profiled() {
#ifdef KIE_PROFILE
  return true;
#else
  return false;
#endif
}

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
