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
  DE_NONFINITE = 4,  // a NaN logit, or a token id outside [0, vocab)
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
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
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
// Tagged words: a float and the epoch it belongs to in one 64-bit word
// (tag << 32 | float bits).  One aligned 64-bit access cannot tear, so a
// reader that sees the tag it waits for has the value too: no fence and no
// separate counter is needed.
__device__ __forceinline__ void st_tagged(unsigned long long *p, float v, uint32_t tag) {
  const unsigned long long w = (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void sred_add(float *p, float v) {
  asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(smem_u32(p)), "f"(v) : "memory");
}
__device__ __forceinline__ void red_add_v4(float *p, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}
// Order-independent fp32 sums (deterministic mode).  A contribution v is
// split into hi = v rounded to a multiple of 2^-8 and lo = (v - hi) rounded
// to a multiple of 2^-25 (|lo| <= 2^-9), each added with ordinary fp32 vector
// atomics into its own accumulator.  With fewer than 256 contributors of
// magnitude below 256, every partial sum of the hi parts is a multiple of
// 2^-8 below 2^16 and every partial sum of the lo parts a multiple of 2^-25
// below 2^-1: both fit fp32's 24-bit significand, so every addition is exact
// and the sums do not depend on the order in which SMs add.  The value read
// back is hi_sum + lo_sum; the rounding of lo costs at most 2^-26 absolute
// per contribution.
constexpr float kHiQ = 256.0f, kHiInvQ = 0.00390625f;                  // 2^8, 2^-8
constexpr float kLoQ = 33554432.0f, kLoInvQ = 2.9802322387695312e-08f;  // 2^25, 2^-25
__device__ __forceinline__ void split_hi_lo(float v, float &hi, float &lo) {
  hi = rintf(v * kHiQ) * kHiInvQ;
  lo = rintf((v - hi) * kLoQ) * kLoInvQ;
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

// Eight weights times eight inputs, as two interleaved fp32 partial sums
// (packed fp32x2 FMAs: one instruction per weight pair).
template <typename T>
__device__ __forceinline__ float2 dot8x2(uint4 w, const float2 (&x)[4], float2 acc) {
  acc = __ffma2_rn(Store<T>::pair(w.x), x[0], acc);
  acc = __ffma2_rn(Store<T>::pair(w.y), x[1], acc);
  acc = __ffma2_rn(Store<T>::pair(w.z), x[2], acc);
  acc = __ffma2_rn(Store<T>::pair(w.w), x[3], acc);
  return acc;
}

// ------------------------------------------------------------------ profiling build
// With -DKIE_PROFILE every SM accumulates SM-clock cycles per activity and
// writes them to KernelArgs::prof[cta * kProfSlots + slot] at exit.
#ifdef KIE_PROFILE
#define KP_BEGIN(var) long long var = (tid == 0) ? clock64() : 0ll
#define KP_END(var, slot) \
  do { if (tid == 0) s.misc->prof[slot] += clock64() - var; } while (0)
// Event trace of one SM over one decode step (thread 0's view): 64-bit words
// (SM clock << 8) | (event type << 4) | argument, into KernelArgs::trace.
#define KT(type, arg) \
  do { if (tracing && tid == 0) trace_put((type), (arg)); } while (0)
#else
#define KP_BEGIN(var) do {} while (0)
#define KP_END(var, slot) do {} while (0)
#define KT(type, arg) do {} while (0)
#endif

// ------------------------------------------------------------------ shared state
struct Misc {
  StageCta sc[ST_COUNT];
  Block blk[kMaxBlocksPerCta];
  __align__(16) float red_sq[4 * kConsumerWarps];  // per-warp sums of squares while staging
  float red_v[kConsumerWarps];
  int32_t red_i[kConsumerWarps];
  volatile int32_t abort;  // a consumer saw a failed wait
  int32_t flag;            // broadcast slot
  long long prof[kProfSlots];
  long long wwait[kConsumerWarps];   // profiling build: tile waits per consumer warp
  int32_t tn;                        // profiling build: trace events recorded
  float fac[4 * 32];   // attention: per-head scale factors of warps or splits
  float hs[8];         // attention: per-head running maximum and sum
  int32_t sel[4];      // sampler: selected digit, keys still needed, keys at the digit, gathered
  float self;          // sampler: broadcast scalar
};

// Scalars of the column stages: the merged attention output of the CTA's KV
// group (at most 4 heads x 128) and the CTA's slice of the SwiGLU hidden units.
constexpr int kSvecO = 512;
constexpr int kSvecFloats = kSvecO + kMaxLocal;

struct Smem {
  uint8_t *ring;
  uint64_t *full, *empty;
  float *vbuf, *part;
  float *svec;   // [0, kSvecO): merged attention output; [kSvecO, ...): hidden slice
  Misc *misc;
};

__device__ __forceinline__ uint32_t *sync_at(const KernelArgs &a, int slot) {
  return a.sync + slot * kSyncStride;
}

__device__ __forceinline__ void raise_error_at(uint32_t *sync, uint32_t code) {
  atomicCAS(sync + SY_STATUS * kSyncStride, 0u, code);
  atomicExch(sync + SY_ABORT * kSyncStride, 1u);
}
__device__ __forceinline__ void raise_error(const KernelArgs &a, uint32_t code) { raise_error_at(a.sync, code); }

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
    const long long el = clock64() - t0;
    pump(el);
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

// Bounded wait until the tagged word *p carries `tag`; its value goes to
// out.  False on watchdog expiry or abort (sync: the counters' base).
__device__ __forceinline__ bool wait_tagged_at(uint32_t *sync, uint64_t watchdog_ns,
                                               const unsigned long long *p, uint32_t tag,
                                               uint32_t where, float &out) {
  unsigned long long w = ld_relaxed_u64(p);
  if (uint32_t(w >> 32) != tag) {
    const long long t0 = clock64(), limit = (long long)watchdog_ns * 2;
    long long next_poll = kAbortPollCycles;
    const uint32_t *abortp = sync + SY_ABORT * kSyncStride;
    for (;;) {
      w = ld_relaxed_u64(p);
      if (uint32_t(w >> 32) == tag) break;
      const long long el = clock64() - t0;
      if (el > next_poll) {
        next_poll = el + kAbortPollCycles;
        if (ld_relaxed(abortp)) return false;
        if (el > limit) {
          raise_error_at(sync, DE_TIMEOUT_COUNTER | (where << 8));
          return false;
        }
      }
    }
  }
  out = __uint_as_float(uint32_t(w));
  return true;
}
__device__ __forceinline__ bool wait_tagged(const KernelArgs &a, const unsigned long long *p, uint32_t tag,
                                            uint32_t where, float &out) {
  return wait_tagged_at(a.sync, a.watchdog_ns, p, tag, where, out);
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
    const long long el = clock64() - t0;
    pump(el);
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

// ------------------------------------------------------------------ kernel instances
// Code that never runs still shapes the persistent loop's register allocation
// and code layout.  Measured on workload 1 (2.3B-class, 128 steps, three
// repeats on one GPU): with the lane-model and ablation branches compiled out
// the dense greedy loop ran 3.0 % faster (892 vs 866 tok/s), and it ran 1.7 %
// faster without the sampler compiled in.  So a launch picks one of these
// instances:
//   dense   (V 0): one lane, dependency counters, fp32 atomic sums, no L2
//           look-ahead -- the decode every dense model runs;
//   lanes   (KV_LANES): the same for lane models (delayed cross-lane mix);
//   general (KV_GENERAL): lane models, the grid-barrier and exact-sum
//           ablations and the L2 look-ahead as runtime switches;
// dense and general with the sampler (KV_SAMPLE) or without it.
// The dense greedy instance is also built for fixed shapes: the attention's
// (query heads per KV head, head size) and the GEMV tile widths of the q/k/v
// stage, of the other row stages and of the column stages.  With them
// constant the attention's per-head loops fold and only the GEMV variants in
// use are compiled, so registers shrink (workload 1, same-GPU A/B: 891 tok/s
// with runtime shapes, 935 with a constant attention shape, 955 with the
// widths constant too).  The lanes instance exists only in a fixed shape.  A
// launch uses a fixed-shape instance only when every field matches the model
// and its plan; 0 means "read at run time".
enum : int { KV_GENERAL = 1, KV_SAMPLE = 2, KV_LANES = 4 };
template <int V, int GS = 0, int DHS = 0, int CQ = 0, int CR = 0, int CC = 0, int CM = 0>
struct Inst {
  static constexpr bool ablations = (V & KV_GENERAL) != 0;   // grid barrier, exact sums, L2 look-ahead
  static constexpr bool lanes = (V & (KV_GENERAL | KV_LANES)) != 0;
  static constexpr bool sample = (V & KV_SAMPLE) != 0;
  static constexpr int g = GS;    // query heads per KV head
  static constexpr int dh = DHS;  // head size
  static constexpr int cq = CQ;   // 16-byte chunks per lane and row of a q/k/v tile
  static constexpr int cr = CR;   // the same for the other row stages (gate/up, LM head)
  static constexpr int cc = CC;   // output groups per thread of the column stages (O, down)
  static constexpr int cm = CM;   // the row width of the lane-mix stage
};

// ------------------------------------------------------------------ weight producer
// One lane of the producer warp issues the CTA's weight tiles, in the order
// the consumers take them, into the ring: one cp.async.bulk (1-D bulk copy, no
// tensor map, no multicast, L2 evict-first) per tile, completing on the slot's
// full mbarrier, after the slot's empty mbarrier says all 16 consumer warps
// released its previous tile.  Weights do not depend on activations, so the
// stream runs ahead across stage, layer and step boundaries while the
// consumers wait for other SMs.  Its state lives in registers; its waits are
// bounded.
template <int V>
struct Producer {
  using I = Inst<V>;
  const KernelArgs &a;
  Smem s;
  const int cta;
  uint32_t T = 0;        // tiles issued
  // L2 look-ahead: bytes of the stream beyond `cur` already requested into L2,
  // and the stream's extent in the current step (it wraps to the start of the
  // stream, the next step's first tile, at `end`).
  uint32_t pf_ahead = 0;
  const uint8_t *base = nullptr, *end = nullptr;
  __device__ Producer(const KernelArgs &a_, Smem s_, int cta_) : a(a_), s(s_), cta(cta_) {}

  // Called while the producer waits for a free ring slot.  A wait longer than
  // l2pf_delay cycles means the consumers are held up by a dependency (other
  // SMs, the attention), not by weights, and HBM would idle; then the next
  // tiles of the stream are requested into L2, one every l2pf_pace cycles, up
  // to l2pf_tiles tiles beyond the ring, so that they land from L2 once the
  // consumers resume.
  __device__ __forceinline__ void l2_lookahead(long long el, uint32_t &nthis, const uint8_t *cur) {
    if (el < a.l2pf_delay + (long long)nthis * a.l2pf_pace) return;
    if (pf_ahead >= uint32_t(a.l2pf_tiles) * kSlotBytes) return;
    const uint8_t *p = cur + pf_ahead;
    if (p >= end) p = base + (p - end);
    if (p >= end) return;
    const uint32_t bytes = uint32_t(min((long long)kSlotBytes, (long long)(end - p)));
    prefetch_l2(p, bytes);
    pf_ahead += bytes;
    ++nthis;
  }

  // The cached K/V rows this CTA's attention split reads in layer l of step
  // `step` (positions before the step's own), pulled into L2 when the layer's
  // first weight tile is issued, well before the attention needs them.
  __device__ void prefetch_kv(int step, int l) const {
    const int Hkv = a.n_kv_heads, g = cta % Hkv, split = cta / Hkv;
    const int nsplit = min((a.n_ctas - 1 - g) / Hkv + 1, kMaxSplit);
    if (split >= nsplit) return;
    const int pos = a.pos0 + step, Lctx = pos + 1;
    const int j0 = int((int64_t)split * Lctx / nsplit);
    const int j1 = min(int((int64_t)(split + 1) * Lctx / nsplit), pos);
    if (j1 <= j0) return;
    const size_t row = ((size_t(l) * Hkv + g) * a.max_seq + j0) * a.head_dim;
    const uint32_t bytes = uint32_t(j1 - j0) * uint32_t(a.head_dim) * 2u;
    prefetch_l2(a.kcache + row, bytes);
    prefetch_l2(a.vcache + row, bytes);
  }

  // Issues every tile of stage k in the order the consumers take them: for a
  // row stage, the column tiles of each row block (rows * 256 cps bytes
  // each); for a column stage, R whole rows of each block at a time.  False
  // once a wait for a free slot gave up.
  __device__ bool stage(int k, const uint8_t *&cur, uint32_t &slot, uint32_t &phase) {
    const StageCta &c = s.misc->sc[k];
    const StageShape &sh = a.shape[k];
    const bool rows = !sh.cols;
    const int nb = rows ? c.nrb : c.nblk, b0 = rows ? c.rb_begin : c.blk_begin;
    const uint32_t rowb = uint32_t(sh.K) * 2u;
    const uint32_t NS = a.ring_slots;
    const int nk = rows ? sh.K / (128 * sh.cps) : 0;
    for (int bi = 0; bi < nb; ++bi) {
      const int nrows = s.misc->blk[b0 + bi].nrows;
      const int ntile = rows ? (nrows > 0 ? nk : 0) : (nrows + sh.R - 1) / sh.R;
      for (int t = 0; t < ntile; ++t) {
        if (T >= NS) {
#ifdef KIE_PROFILE
          const long long tw = clock64();
#endif
          // the slot's previous tile (T - NS) was released by every consumer warp
          uint32_t nthis = 0;
          const uint8_t *c0 = cur;
          const bool pf = I::ablations && a.l2pf_tiles > 0;
          if (!wait_mbar(a, &s.empty[slot], phase ^ 1u, DE_TIMEOUT_EMPTY, [&](long long el) {
                if (pf) l2_lookahead(el, nthis, c0);
              }))
            return false;
#ifdef KIE_PROFILE
          s.misc->prof[PF_PROD_EMPTY] += clock64() - tw;
#endif
        }
        const uint32_t bytes = rows ? uint32_t(nrows) * 256u * uint32_t(sh.cps)
                                    : uint32_t(min(sh.R, nrows - t * sh.R)) * rowb;
        mbar_expect_tx(&s.full[slot], bytes);
        bulk_g2s(s.ring + size_t(slot) * kSlotBytes, cur, bytes, &s.full[slot], policy_evict_first());
        cur += bytes;
        pf_ahead = pf_ahead > bytes ? pf_ahead - bytes : 0u;
        ++T;
        if (++slot == NS) { slot = 0; phase ^= 1u; }
      }
    }
    return true;
  }

  __device__ void run() {
    base = a.wstream + a.cta_stream_off[cta];
    const bool lanes = I::lanes && a.n_lanes > 1;
    // bytes of one step's stream: every layer's stages, then the final lane
    // mix and the LM head (when the step computes logits)
    const StageCta *sc = s.misc->sc;
    const int64_t layer_bytes = sc[ST_QKV].bytes + sc[ST_O].bytes + sc[ST_GU].bytes + sc[ST_D].bytes;
    const int64_t body = int64_t(a.n_layers) * layer_bytes +
                         (lanes ? int64_t(a.n_layers - 1) * sc[ST_MIX].bytes : 0);
    const int64_t head = (lanes ? sc[ST_MIX].bytes : 0) + sc[ST_LM].bytes;
    uint32_t slot = 0, phase = 0;   // phase: parity of the slot's current use
    bool ok = true;
    for (int step = 0; step < a.n_steps && ok; ++step) {
      const uint8_t *cur = base;
      const bool lm = a.logits_every_step || step == a.n_steps - 1;
      end = base + body + (lm ? head : 0);
      for (int l = 0; l < a.n_layers && ok; ++l) {
        prefetch_kv(step, l);
        ok = stage(ST_QKV, cur, slot, phase);
        if (ok && lanes && l >= 1) ok = stage(ST_MIX, cur, slot, phase);
        ok = ok && stage(ST_O, cur, slot, phase);
        ok = ok && stage(ST_GU, cur, slot, phase);
        ok = ok && stage(ST_D, cur, slot, phase);
      }
      if (ok && (a.logits_every_step || step == a.n_steps - 1)) {
        if (lanes) ok = stage(ST_MIX, cur, slot, phase);
        ok = ok && stage(ST_LM, cur, slot, phase);
      }
    }
    drain();
  }

  // Before the CTA exits: each slot holds at most one outstanding copy, the
  // last one issued into it; wait (bounded) until those have landed.
  __device__ void drain() const {
    const uint32_t NS = a.ring_slots;
    const uint32_t first = T > NS ? T - NS : 0;
    for (uint32_t t = first; t < T; ++t) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&s.full[t % NS], (t / NS) & 1))
        if (clock64() - t0 > (long long)a.watchdog_ns * 2) break;
    }
  }
};

// ---- logit keys: (order-preserving bits of the value) << 32 | (~row), so
// that a larger key is a larger logit, and among equal logits the lower
// row; every finite or infinite logit's key is above 0.  -0 and +0 are
// equal logits, so both take +0's bits (else +0 would outrank -0).
__device__ __forceinline__ unsigned long long logit_key(float v, int row) {
  const uint32_t fb = __float_as_uint(v == 0.f ? 0.f : v);
  const uint32_t ord = (fb & 0x80000000u) ? ~fb : (fb | 0x80000000u);
  return (static_cast<unsigned long long>(ord) << 32) | (0xffffffffu - uint32_t(row));
}
__device__ __forceinline__ float key_value(unsigned long long key) {
  const uint32_t ord = uint32_t(key >> 32);
  return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}
__device__ __forceinline__ int key_row(unsigned long long key) {
  return int(0xffffffffu - uint32_t(key & 0xffffffffull));
}

// ------------------------------------------------------------------ sampling
// Sampling beyond greedy (temperature, top-k, top-p; the uniform of each step
// is an input).  Every CTA computes the same token from the same global data,
// so no further exchange is needed once it is drawn.  These run once per
// token and exist only in the sampling instance of the kernel.

// What the sampler reads.
struct SampleArgs {
  const float *zbuf;
  unsigned long long *cand, *psum;
  const unsigned long long *keys;
  const float *uniforms;
  const StageCta *stage_cta;
  uint32_t *sync;
  uint64_t watchdog_ns;
  float t, p;                // temperature, top-p
  int32_t k, vocab, n_ctas;  // top-k
};

// Before the token barrier, top-k mode: this CTA's sample_k largest logit
// keys, largest first, into cand[cta] (its LM-head rows' keys, read back
// from zbuf and sorted in shared memory by a descending bitonic sort; 0
// pads a slice shorter than k).
__device__ __forceinline__ void local_topk(const SampleArgs g, const Smem s, int tid, int cta) {
  const StageCta &c = s.misc->sc[ST_LM];
  const int n = c.nout;
  int np = 2;
  while (np < n) np <<= 1;   // n <= kMaxSampleRows (checked on the host): fits `part`
  unsigned long long *kp = reinterpret_cast<unsigned long long *>(s.part);
  for (int i = tid; i < np; i += kNC)
    kp[i] = i < n ? logit_key(__ldcg(g.zbuf + c.row0 + i), c.row0 + i) : 0ull;
  cbar();
  for (int size = 2; size <= np; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < np; i += kNC) {
        const int j = i ^ stride;
        if (j > i) {
          const unsigned long long x = kp[i], y = kp[j];
          if ((i & size) == 0 ? x < y : x > y) { kp[i] = y; kp[j] = x; }
        }
      }
      cbar();
    }
  for (int j = tid; j < g.k; j += kNC)
    g.cand[size_t(cta) * kMaxTopK + j] = j < n ? kp[j] : 0ull;
}

// After the token barrier, top-k mode.  The k = min(sample_k, V) largest
// keys of all CTAs' candidates: a radix select over 8-bit digits from the
// top keeps a prefix and the number of keys still needed below it, and
// stops once the keys sharing the prefix are exactly those; the kept keys
// are gathered and ranked (largest first) in shared memory.  Thread 0 then
// weighs them exp((z - z_max) / T), cuts the most probable leading set
// reaching top_p of their sum, and draws by inverse CDF in token order.
__device__ __forceinline__ int sample_topk(const SampleArgs g, const Smem s, int tid, int step) {
  const int warp = tid >> 5, lane = tid & 31;
  const int kc = g.k, k = min(kc, g.vocab), total = g.n_ctas * kc;
  uint32_t *hist = reinterpret_cast<uint32_t *>(s.part);                 // [256]
  unsigned long long *sel = reinterpret_cast<unsigned long long *>(s.part + 256);  // [kMaxTopK]
  unsigned long long *srt = sel + kMaxTopK;                              // [kMaxTopK]
  float *ev = reinterpret_cast<float *>(srt + kMaxTopK);                 // [kMaxTopK]
  int *byrow = reinterpret_cast<int *>(ev + kMaxTopK);                   // [kMaxTopK]
  auto cand_at = [&](int q) { return __ldcg(g.cand + size_t(q / kc) * kMaxTopK + q % kc); };
  unsigned long long prefix = 0, mask = 0;
  int need = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kNC) hist[i] = 0;
    cbar();
    for (int q = tid; q < total; q += kNC) {
      const unsigned long long key = cand_at(q);
      if (key != 0ull && (key & mask) == prefix) atomicAdd(&hist[uint32_t(key >> shift) & 255u], 1u);
    }
    cbar();
    if (warp == 0) {
      // lane l holds bins 255 - 8 l - e (e < 8): lane 0 the highest digits
      uint32_t h[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { h[e] = hist[255 - 8 * lane - e]; tot += h[e]; }
      uint32_t incl = tot;
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const uint32_t above = incl - tot;
      if (above < uint32_t(need) && uint32_t(need) <= incl) {   // exactly one lane
        uint32_t acc = above;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (acc + h[e] >= uint32_t(need)) {
            s.misc->sel[0] = 255 - 8 * lane - e;
            s.misc->sel[1] = need - int(acc);
            s.misc->sel[2] = int(h[e]);
            break;
          }
          acc += h[e];
        }
      }
    }
    cbar();
    prefix |= static_cast<unsigned long long>(s.misc->sel[0]) << shift;
    mask |= 0xffull << shift;
    need = s.misc->sel[1];
    const bool done = s.misc->sel[2] == need;   // every key with this prefix is taken
    cbar();
    if (done) break;
  }
  if (tid == 0) s.misc->sel[3] = 0;
  cbar();
  for (int q = tid; q < total; q += kNC) {
    const unsigned long long key = cand_at(q);
    if (key != 0ull && (key & mask) >= prefix) {
      const int slot = atomicAdd(&s.misc->sel[3], 1);
      if (slot < kMaxTopK) sel[slot] = key;
    }
  }
  cbar();
  const int m = min(s.misc->sel[3], kMaxTopK);   // k, the keys being distinct
  if (tid < m) {
    const unsigned long long x = sel[tid];
    int r = 0;
    for (int i = 0; i < m; ++i) r += sel[i] > x;
    srt[r] = x;
  }
  cbar();
  if (tid == 0) {
    const float zmax = key_value(srt[0]), temp = g.t;
    float S = 0.f;
    for (int j = 0; j < m; ++j) {
      ev[j] = expf((key_value(srt[j]) - zmax) / temp);
      S += ev[j];
    }
    int mm = m;
    if (g.p < 1.f) {   // most probable first, until top_p of the mass
      const float lim = g.p * S;
      float c = 0.f;
      mm = 0;
      do { c += ev[mm]; ++mm; } while (mm < m && c < lim);
    }
    s.misc->sel[3] = mm;
  }
  cbar();
  const int mm = s.misc->sel[3];
  if (tid < mm) {
    const int row = key_row(srt[tid]);
    int r = 0;
    for (int i = 0; i < mm; ++i) r += key_row(srt[i]) < row;
    byrow[r] = tid;
  }
  cbar();
  if (tid == 0) {
    float S = 0.f;
    for (int r = 0; r < mm; ++r) S += ev[byrow[r]];
    const float target = __ldg(g.uniforms + step) * S;
    int tk = key_row(srt[byrow[mm - 1]]);
    float c = 0.f;
    for (int r = 0; r < mm; ++r) {
      c += ev[byrow[r]];
      if (c > target) { tk = key_row(srt[byrow[r]]); break; }
    }
    s.misc->sel[0] = tk;
  }
  cbar();
  return s.misc->sel[0];
}

// After the token barrier, no top-k cut (top_p 1): every token, in token
// order.  With z_max from the argmax key, each CTA adds exp((z - z_max) / T)
// over its LM-head rows (a fixed order) and publishes the sum as a tagged
// word; every CTA walks the CTAs' sums in order (their row slices are
// consecutive) to the slice that holds the draw, and warp 0 walks that
// slice's rows: each lane a run of rows, a scan of the runs' sums, then the
// lane whose run crosses walks it.  A crossing lost to rounding falls back
// to the slice's last row.  Returns -1 if a wait gave up.
__device__ __forceinline__ int sample_full(const SampleArgs g, const Smem s, int tid, int cta, int step,
                                        uint32_t lm_count) {
  const int warp = tid >> 5, lane = tid & 31;
  const float zmax = key_value(__ldcg(g.keys + step)), temp = g.t;
  const StageCta &c = s.misc->sc[ST_LM];
  float e = 0.f;
  for (int i = tid; i < c.nout; i += kNC) e += expf((__ldcg(g.zbuf + c.row0 + i) - zmax) / temp);
  for (int o = 16; o; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
  if (lane == 0) s.misc->red_v[warp] = e;
  cbar();
  const uint32_t tag = lm_count;
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kConsumerWarps; ++w) t += s.misc->red_v[w];
    st_tagged(g.psum + cta, t, tag);
  }
  float *ps = s.vbuf;
  bool ok = true;
  for (int q = tid; q < g.n_ctas; q += kNC) ok = ok && wait_tagged_at(g.sync, g.watchdog_ns, g.psum + q, tag, 0x90, ps[q]);
  if (!ok) s.misc->abort = 1;
  cbar();
  if (s.misc->abort != 0) return -1;
  if (tid == 0) {
    float S = 0.f;
    for (int q = 0; q < g.n_ctas; ++q) S += ps[q];
    const float target = __ldg(g.uniforms + step) * S;
    int cs = -1;
    float before = 0.f;
    for (int q = 0; q < g.n_ctas; ++q) {
      if (ps[q] > 0.f) cs = q;
      if (before + ps[q] > target) { cs = q; break; }
      before += ps[q];
    }
    if (cs < 0) cs = g.n_ctas - 1;
    before = 0.f;
    for (int q = 0; q < cs; ++q) before += ps[q];
    s.misc->sel[0] = cs;
    s.misc->self = before;
    ps[g.n_ctas] = target;
  }
  cbar();
  if (warp == 0) {
    const int cs = s.misc->sel[0];
    const float target = ps[g.n_ctas];
    const StageCta sc = g.stage_cta[size_t(ST_LM) * g.n_ctas + cs];
    const int ch = (sc.nout + 31) / 32, i0 = min(lane * ch, sc.nout), i1 = min(i0 + ch, sc.nout);
    float run = 0.f;
    for (int i = i0; i < i1; ++i) run += expf((__ldcg(g.zbuf + sc.row0 + i) - zmax) / temp);
    float incl = run;
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const float base = s.misc->self + (incl - run);
    const unsigned ball = __ballot_sync(0xffffffffu, i1 > i0 && base + run > target);
    int tk = sc.row0 + sc.nout - 1;
    if (ball) {
      const int src = __ffs(ball) - 1;
      int found = sc.row0 + i1 - 1;
      if (lane == src) {
        float cum = base;
        for (int i = i0; i < i1; ++i) {
          cum += expf((__ldcg(g.zbuf + sc.row0 + i) - zmax) / temp);
          if (cum > target) { found = sc.row0 + i; break; }
        }
      }
      tk = __shfl_sync(0xffffffffu, found, src);
    }
    if (lane == 0) s.misc->sel[1] = tk;
  }
  cbar();
  return s.misc->sel[1];
}

// ------------------------------------------------------------------ consumer
template <typename T, int V, int GS, int DHS, int CQ, int CR, int CC, int CM>
struct Consumer {
  using I = Inst<V, GS, DHS, CQ, CR, CC, CM>;
  const KernelArgs &a;
  Smem s;
  const int tid, warp, lane, cta;
  uint32_t Tbase = 0;   // tiles consumed before the current stage
  uint32_t slot = 0, phase = 0;   // ring position of the next tile (every warp sees every tile)
  int step = 0, l = 0, tok = 0, p = 0;
  uint32_t gl = 0;        // global layer index step * n_layers + l (parity of the buffers)
  uint32_t lm_count = 0;
  uint32_t nsig = 0;      // signals this CTA has made (grid-barrier mode)
  bool tracing = false;   // profiling build: this SM records the current step
#ifdef KIE_PROFILE
  __device__ void trace_put(int type, int arg) {
    const int n = s.misc->tn;
    if (n < a.trace_cap) a.trace[1 + n] = (static_cast<unsigned long long>(clock64()) << 8) |
                                          uint32_t(((type & 15) << 4) | (arg & 15));
    s.misc->tn = n + 1;
  }
#endif

  __device__ Consumer(const KernelArgs &a_, Smem s_, int tid_, int cta_)
      : a(a_), s(s_), tid(tid_), warp(tid_ >> 5), lane(tid_ & 31), cta(cta_) {}

  __device__ bool aborted() const { return s.misc->abort != 0; }
  // attention shape: compile-time in the shape-specialised instances
  __device__ __forceinline__ int head_dim() const { return I::dh ? I::dh : a.head_dim; }
  __device__ __forceinline__ int group() const { return I::g ? I::g : a.n_heads / a.n_kv_heads; }

  // thread 0 waits for a counter, everyone learns the outcome.  In grid-barrier
  // mode (an ablation of the per-dependency counters) every wait is instead
  // for all CTAs to have made as many signals as this one: every CTA makes the
  // same sequence of signals, and each gate follows the signal it waits for.
  __device__ bool gate(int slot, uint32_t target, uint32_t where, int pkind) {
    if (tid == 0) {
#ifdef KIE_PROFILE
      const long long t0 = clock64();
#endif
      if (I::ablations && a.grid_sync) {
        slot = SY_GRID;
        target = nsig * a.n_ctas;
      }
      KT(TE_GATE_BEGIN, pkind);
      if (!wait_counter(a, sync_at(a, slot), target, where, [](long long) {})) s.misc->abort = 1;
      KT(TE_GATE_END, pkind);
#ifdef KIE_PROFILE
      s.misc->prof[PF_GATE] += clock64() - t0;
      s.misc->prof[PF_GATE_K + pkind] += clock64() - t0;
      s.misc->prof[PF_NGATE] += 1;
#endif
    }
    cbar();
    return !aborted();
  }

  __device__ void signal(int slot) {
    KP_BEGIN(t_sig);
    KT(TE_SIGNAL_BEGIN, 0);
    cbar();
    KT(TE_SIGNAL_END, 0);
    ++nsig;
    if (tid == 0) red_release_add(sync_at(a, (I::ablations && a.grid_sync) ? int(SY_GRID) : slot), 1u);
    KP_END(t_sig, PF_SIGNAL);
  }

  // ---- stage inputs
  __device__ static float4 add4(float4 u, float4 v) {
    return make_float4(u.x + v.x, u.y + v.y, u.z + v.z, u.w + v.w);
  }
  __device__ const float4 *vec4(const float *base, uint32_t parity) const {
    return reinterpret_cast<const float4 *>(base + size_t(parity & 1u) * a.d_model);
  }
  // Elements 4j..4j+3 of a layer accumulator (acc_o or acc_d) of the given
  // parity: the fp32 sums, or in deterministic mode the hi sums plus the lo
  // sums (stored 2 d floats further on).
  __device__ float4 acc4(const float *base, uint32_t parity, int j) const {
    const float4 h = __ldcg(vec4(base, parity) + j);
    if (!(I::ablations && a.det_sum)) return h;
    const float4 l = __ldcg(vec4(base + 2 * size_t(a.d_model), parity) + j);
    return make_float4(h.x + l.x, h.y + l.y, h.z + l.z, h.w + l.w);
  }
  // Adds outputs e .. e+3 into a layer accumulator of the given parity.
  __device__ __forceinline__ void acc_add4(float *base, uint32_t parity, int e, float4 v) const {
    float *p = base + size_t(parity & 1u) * a.d_model + e;
    if (!(I::ablations && a.det_sum)) {
      red_add_v4(p, v);
      return;
    }
    float4 hi, lo;
    split_hi_lo(v.x, hi.x, lo.x);
    split_hi_lo(v.y, hi.y, lo.y);
    split_hi_lo(v.z, hi.z, lo.z);
    split_hi_lo(v.w, hi.w, lo.w);
    red_add_v4(p, hi);
    red_add_v4(p + 2 * size_t(a.d_model), lo);
  }
  // elements 4j..4j+3 of the residual entering the current layer (the
  // embedding row at layer 0), plus the delayed cross-lane sum landing here
  __device__ float4 xin4(int j) const {
    float4 v;
    if (l == 0) {
      const uint2 w = *reinterpret_cast<const uint2 *>(a.embed + size_t(tok) * a.d_model + 4 * j);
      const float2 lo = Store<T>::pair(w.x), hi = Store<T>::pair(w.y);
      v = make_float4(lo.x, lo.y, hi.x, hi.y);
    } else {
      const uint32_t q = gl - 1;
      v = add4(add4(__ldcg(vec4(a.xres, q) + j), acc4(a.acc_o, q, j)), acc4(a.acc_d, q, j));
    }
    if (I::lanes && a.n_lanes > 1 && l >= a.lane_delay)
      v = add4(v, __ldcg(reinterpret_cast<const float4 *>(
                             a.dsum + size_t((l - a.lane_delay) % a.lane_delay) * a.d_model) + j));
    return v;
  }

  // Staging of a row stage's input: vbuf[0..n) = src(i) * gain[i] (gain may
  // be null: no gain), and red_sq[i] = the sum of src^2 over elements
  // [128 i, 128 i + 128), so that the mean square of any lane slice (a
  // multiple of 128 elements) is a sum of red_sq entries.  The RMSNorm's
  // scalar factor rsqrt(mean(x^2) + eps) commutes with the dot products and
  // is applied to the row sums (norm_scale).  src(j) returns elements
  // 4j .. 4j+3.  If own is not null, this CTA's rows [own_lo, own_hi) of the
  // raw input are also written to own (the residual kept by its row owners).
  template <typename Src>
  __device__ void stage_input(Src src, const float *gain, int n, float *own = nullptr,
                              int own_lo = 0, int own_hi = 0) {
    KP_BEGIN(t_norm);
    KT(TE_NORM_BEGIN, 0);
    const int ng = n >> 2;
    float4 *vb = reinterpret_cast<float4 *>(s.vbuf);
    for (int q = 0; q * kNC < ng; ++q) {
      const int j = tid + q * kNC;
      float ss = 0.f;
      if (j < ng) {
        const float4 v = src(j);
        if (own && 4 * j + 3 >= own_lo && 4 * j < own_hi) {
          const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (4 * j + u >= own_lo && 4 * j + u < own_hi) own[4 * j + u] = e[u];
        }
        const float4 g = gain ? __ldg(reinterpret_cast<const float4 *>(gain) + j)
                              : make_float4(1.f, 1.f, 1.f, 1.f);
        vb[j] = make_float4(v.x * g.x, v.y * g.y, v.z * g.z, v.w * g.w);
        ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s.misc->red_sq[q * kConsumerWarps + warp] = ss;
    }
    cbar();
    KT(TE_NORM_END, 0);
    KP_END(t_norm, PF_STAGE);
  }

  // rsqrt(mean(x^2) + eps) over the norm slice [in_off, in_off + seg) of the
  // staged input (seg = 0: no norm, factor 1).
  __device__ float norm_scale(int in_off, int seg) const {
    if (seg == 0) return 1.f;
    float tot = 0.f;
    for (int i = in_off >> 7; i < (in_off + seg) >> 7; ++i) tot += s.misc->red_sq[i];
    return rsqrtf(tot / float(seg) + a.rms_eps);
  }

  // Waits (warp-wide outcome) for the weight tile in the current ring slot.
  __device__ __forceinline__ bool tile_wait(int k) {
    bool got = true;
    KT(TE_TILE_WAIT, 0);
    if (lane == 0) got = wait_mbar(a, &s.full[slot], phase, DE_TIMEOUT_FULL | (k << 8), [](long long) {});
    KT(TE_TILE_READY, 0);
    return __shfl_sync(0xffffffffu, got, 0);
  }
  // Hands ring slot `sl` back to the producer as soon as this warp has
  // loaded its words from it: __syncwarp orders every lane's loads before
  // lane 0's arrive, whose release semantics order them before the producer
  // can observe the arrival and overwrite the slot.
  __device__ __forceinline__ void release_slot(uint32_t sl) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[sl]);
  }
  __device__ void slot_advance() {
    if (++slot == uint32_t(a.ring_slots)) { slot = 0; phase ^= 1u; }
  }

  // ---- row stages: out(local row, (W[row, :] . vin) * norm factor)
  // For each row block (at most 128 / C rows with one input slice): lane l
  // takes rows l + 32 j; warp w takes the 16-byte chunks w C .. w C + C - 1 of
  // every tile (8 C columns), found at chunk position ^ (row & 7).  A warp
  // loads its words of a tile, hands the slot back, then does the tile's
  // arithmetic; its rows' partial dot products stay in registers across the
  // block's tiles (no reduction per tile, so the 16 warps working on a tile
  // keep its short load latency covered).  At the end of the block each warp
  // writes its partials (double-buffered by block parity), one barrier, and
  // the block's row sums are the 16 warps' partials added in warp order
  // (deterministic), scaled by the block's RMSNorm factor and handed to out()
  // by thread `row`.  Ends with a barrier, so out()'s shared-memory results
  // are visible to every consumer thread.
  template <int C>
  struct RowWords {
    uint4 q[4 / C][C];
  };

  template <int C>
  __device__ __forceinline__ RowWords<C> row_fetch(int k, int nrows, uint32_t &sl, bool &ok) {
    constexpr int JM = 4 / C;
    constexpr int KB2 = 256 * C;   // bytes of one tile row
    RowWords<C> w;
    sl = slot;
    ok = ok && tile_wait(k);
    const uint8_t *tile = s.ring + size_t(slot) * kSlotBytes;
#pragma unroll
    for (int j = 0; j < JM; ++j) {
      const int r = lane + 32 * j;
      const bool in = ok && r < nrows;
#pragma unroll
      for (int cc = 0; cc < C; ++cc)
        w.q[j][cc] = in ? *reinterpret_cast<const uint4 *>(tile + r * KB2 + (((warp * C + cc) ^ (r & 7)) << 4))
                        : make_uint4(0u, 0u, 0u, 0u);
    }
    slot_advance();
    return w;
  }

  template <int C>
  __device__ __forceinline__ void row_math(const RowWords<C> &w, const float *xin, float2 (&acc)[4 / C]) const {
    constexpr int JM = 4 / C;
#pragma unroll
    for (int cc = 0; cc < C; ++cc) {
      const float4 x0 = *reinterpret_cast<const float4 *>(xin + 8 * cc);
      const float4 x1 = *reinterpret_cast<const float4 *>(xin + 8 * cc + 4);
      const float2 xv[4] = {make_float2(x0.x, x0.y), make_float2(x0.z, x0.w),
                            make_float2(x1.x, x1.y), make_float2(x1.z, x1.w)};
#pragma unroll
      for (int j = 0; j < JM; ++j) acc[j] = dot8x2<T>(w.q[j][cc], xv, acc[j]);
    }
  }

  template <int C, typename OutF>
  __device__ void gemv_rows_c(int k, const float *vin, OutF &out) {
    constexpr int JM = 4 / C;
    constexpr int KB = 128 * C;
    const StageCta &c = s.misc->sc[k];
    const int nk = a.shape[k].K / KB, seg = a.shape[k].norm;
    bool ok = !aborted();
    for (int rb = 0; rb < c.nrb; ++rb) {
      const Block b = s.misc->blk[c.rb_begin + rb];
      const float *xw = vin + b.in_off + warp * 8 * C;   // this warp's columns of tile 0
      float2 acc[JM];
#pragma unroll
      for (int j = 0; j < JM; ++j) acc[j] = make_float2(0.f, 0.f);
      for (int t = 0; t < nk && ok; ++t) {
        uint32_t sl = 0;
        const RowWords<C> w = row_fetch<C>(k, b.nrows, sl, ok);
        if (!ok) break;
        release_slot(sl);
        row_math<C>(w, xw + t * KB, acc);
        KT(TE_TILE_DONE, 0);
      }
      float *pb = s.part + (rb & 1) * (kConsumerWarps * kMaxRowBlock);
#pragma unroll
      for (int j = 0; j < JM; ++j)
        if (lane + 32 * j < b.nrows) pb[warp * kMaxRowBlock + lane + 32 * j] = acc[j].x + acc[j].y;
      cbar();
      if (tid < b.nrows) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) v += pb[w * kMaxRowBlock + tid];
        out(b.lrow0 + tid, v * norm_scale(b.in_off, seg));
      }
    }
    if (!ok) s.misc->abort = 1;
    cbar();
  }

  template <typename OutF>
  __device__ void gemv_rows(int k, const float *vin, OutF &&out) {
    KP_BEGIN(t_gemv);
    KT(TE_STAGE_BEGIN, k);
    // call sites pass a constant k
    const int fixed = k == ST_QKV ? I::cq : k == ST_MIX ? I::cm : I::cr;
    switch (fixed ? fixed : a.shape[k].cps) {
      case 4: gemv_rows_c<4>(k, vin, out); break;
      case 2: gemv_rows_c<2>(k, vin, out); break;
      default: gemv_rows_c<1>(k, vin, out); break;
    }
    Tbase += s.misc->sc[k].ntiles;
    KT(TE_STAGE_END, k);
    KP_END(t_gemv, k == ST_LM ? PF_LM : PF_GEMV);
    KP_END(t_gemv, PF_GEMV_K + k);
  }

  // Row sums of the last non-LM row stage, kept in shared memory.
  __device__ float *rsum() const { return s.part + a.rsum_off; }

  // ---- attention over the cache for one KV head group (split-KV)
  // Positions of this CTA's split: [j0, j1) of 0..p.  Each warp folds
  // positions j0 + warp + W*i, two per iteration.
  static constexpr int kU = 2;
  struct KvWords {
    uint2 k[kU], v[kU];   // raw storage words of this lane (dh 64 uses .x only)
  };
  __device__ void kv_range(int &j0, int &j1, int &split, int &nsplit) const {
    const int Hkv = a.n_kv_heads, g = cta % Hkv;
    split = cta / Hkv;
    const int ngroup = (a.n_ctas - 1 - g) / Hkv + 1;      // CTAs of this KV group
    nsplit = min(ngroup, kMaxSplit);                      // those that take positions
    const int Lctx = p + 1;
    j0 = split < nsplit ? int((int64_t)split * Lctx / nsplit) : 0;
    j1 = split < nsplit ? int((int64_t)(split + 1) * Lctx / nsplit) : 0;
  }
  // Loads the cached K/V rows of positions jb + u*W (u < kU) that lie in
  // [jb, j1) and before p (row p is written in this step and comes from
  // shared memory instead).
  __device__ void kv_load(KvWords &w, int jb, int j1) const {
    const int dh = head_dim(), Hkv = a.n_kv_heads, g = cta % Hkv;
    const size_t base = ((size_t(l) * Hkv + g) * a.max_seq) * dh;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = jb + u * kConsumerWarps;
      w.k[u] = make_uint2(0u, 0u);
      w.v[u] = make_uint2(0u, 0u);
      if (j < j1 && j != p) {
        if (dh == 128) {
          w.k[u] = __ldcg(reinterpret_cast<const uint2 *>(a.kcache + base + size_t(j) * dh) + lane);
          w.v[u] = __ldcg(reinterpret_cast<const uint2 *>(a.vcache + base + size_t(j) * dh) + lane);
        } else {
          w.k[u].x = __ldcg(reinterpret_cast<const unsigned int *>(a.kcache + base + size_t(j) * dh) + lane);
          w.v[u].x = __ldcg(reinterpret_cast<const unsigned int *>(a.vcache + base + size_t(j) * dh) + lane);
        }
      }
    }
  }
  __device__ void attention() {
    KP_BEGIN(t_attn);
    KT(TE_ATTN, 0);
    attention_body();
    KT(TE_ATTN, 3);
    KP_END(t_attn, PF_ATTN);
  }

  // RoPE of this step's q (scaled by 1/sqrt(dh)) and k, k and v rounded to
  // the cache type (the current token uses the rounded values too), into
  // shared memory: qs [G][dh], kcur [dh], vcur [dh] at the start of vbuf.
  // The writer also stores position p's K/V in the cache.  Ends with a
  // barrier.
  __device__ void attn_prologue(bool writer) {
    const int dh = head_dim(), half = dh >> 1;
    const int Hkv = a.n_kv_heads, G = group();
    const int g = cta % Hkv;
    float *qs = s.vbuf;
    float *kcur = qs + G * dh;
    float *vcur = kcur + dh;
    const float2 *cs = a.rope_cs + size_t(p) * half;
    const size_t cache_row = ((size_t(l) * Hkv + g) * a.max_seq + p) * dh;
    // q/k/v of this layer are tagged gl + 1 by the SMs that computed them;
    // every thread waits for the words it reads
    const uint32_t tag = gl + 1;
    bool ok = true;
    for (int idx = tid; idx < (G + 2) * dh; idx += kNC) {
      const int hh = idx / dh, d = idx - hh * dh;
      const int dd = d < half ? d : d - half;
      const float2 c = cs[dd];
      // row of the fused q/k/v output: query head g G + hh, or the group's k or v
      const size_t row = hh < G ? size_t(g * G + hh) * dh
                                : (hh == G ? size_t(a.n_heads) * dh : size_t(a.n_heads + Hkv) * dh) +
                                      size_t(g) * dh;
      float v0 = 0.f, v1 = 0.f;
      ok = ok && wait_tagged(a, a.qkv + row + d, tag, 0x20, v0);
      if (hh <= G) ok = ok && wait_tagged(a, a.qkv + row + (d < half ? d + half : d - half), tag, 0x20, v1);
      if (hh < G) {
        const float r = d < half ? v0 * c.x - v1 * c.y : v0 * c.x + v1 * c.y;
        qs[idx] = r * a.attn_scale;
      } else if (hh == G) {
        const float r = d < half ? v0 * c.x - v1 * c.y : v0 * c.x + v1 * c.y;
        const uint16_t b = Store<T>::from_f(r);
        kcur[d] = Store<T>::to_f(b);
        if (writer && ok) a.kcache[cache_row + d] = b;
      } else {
        const uint16_t b = Store<T>::from_f(v0);
        vcur[d] = Store<T>::to_f(b);
        if (writer && ok) a.vcache[cache_row + d] = b;
      }
    }
    if (!ok) s.misc->abort = 1;
    cbar();
  }

  __device__ void attention_body() {
    const int dh = head_dim();
    const int Hkv = a.n_kv_heads, G = group();
    const int g = cta % Hkv;
    int j0, j1, split, nsplit;
    kv_range(j0, j1, split, nsplit);
    // the first cached rows (already pulled into L2 by the producer) are
    // requested together with this step's q/k/v
    KvWords kw;
    kv_load(kw, j0 + warp, j1);
    const bool active = split < nsplit;
    const bool writer = (split == nsplit - 1);  // its range holds position p
    const uint32_t tag = gl + 1;                // this layer's tag of exchanged words
    float *qs = s.vbuf;              // [G][dh] roped, scaled queries
    float *kcur = qs + G * dh;       // [dh] roped, rounded key of position p
    float *vcur = kcur + dh;         // [dh] rounded value of position p
    float *wst = vcur + dh;          // [W][G][dh + 2] per-warp softmax states
    attn_prologue(writer);
    if (aborted()) return;
    // Online softmax, kU positions per iteration: their score reductions are
    // independent and one rescale covers them.  The next iteration's rows are
    // requested before this one's arithmetic.
    const int dpl = dh >> 5;  // dims per lane: 4 (dh 128) or 2 (dh 64)
    float m[4], lsum[4], o[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[i] = -INFINITY;
      lsum[i] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    }
    constexpr int U = kU;
    for (int jb = j0 + warp; jb < j1; jb += U * kConsumerWarps) {
      float kv[U][4], vv[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = jb + u * kConsumerWarps;
        if (j == p) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kv[u][e] = e < dpl ? kcur[lane * dpl + e] : 0.f;
            vv[u][e] = e < dpl ? vcur[lane * dpl + e] : 0.f;
          }
        } else {
          float2 f;
          f = Store<T>::pair(kw.k[u].x); kv[u][0] = f.x; kv[u][1] = f.y;
          f = Store<T>::pair(kw.k[u].y); kv[u][2] = f.x; kv[u][3] = f.y;
          f = Store<T>::pair(kw.v[u].x); vv[u][0] = f.x; vv[u][1] = f.y;
          f = Store<T>::pair(kw.v[u].y); vv[u][2] = f.x; vv[u][3] = f.y;
        }
      }
      kv_load(kw, jb + U * kConsumerWarps, j1);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i < G) {
          float sc[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            float t = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < dpl) t = fmaf(qs[i * dh + lane * dpl + e], kv[u][e], t);
            sc[u] = t;
          }
#pragma unroll
          for (int of = 16; of; of >>= 1)
#pragma unroll
            for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], of);
          float mx = m[i];
#pragma unroll
          for (int u = 0; u < U; ++u)
            if (jb + u * kConsumerWarps < j1) mx = fmaxf(mx, sc[u]);
          const float corr = expf(m[i] - mx);
          float pu[U], ps = 0.f;
#pragma unroll
          for (int u = 0; u < U; ++u) {
            pu[u] = (jb + u * kConsumerWarps < j1) ? expf(sc[u] - mx) : 0.f;
            ps += pu[u];
          }
          lsum[i] = lsum[i] * corr + ps;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float acc = o[i][e] * corr;
#pragma unroll
            for (int u = 0; u < U; ++u) acc = fmaf(pu[u], vv[u][e], acc);
            o[i][e] = acc;
          }
          m[i] = mx;
        }
      }
    }
    KT(TE_ATTN, 1);
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
    // combine the warps into this CTA's partial for each query head: warp i
    // finds head i's running maximum over the 16 warps and each warp's scale
    // factor once; then every output element is a 16-term weighted sum
    float *fac = s.misc->fac, *hs = s.misc->hs;
    if (warp < G) {
      const int i = warp;
      const float mw = lane < kConsumerWarps ? wst[(size_t(lane) * G + i) * st + dh] : -INFINITY;
      float M = mw;
      for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float f = mw == -INFINITY ? 0.f : expf(mw - M);
      float L = lane < kConsumerWarps ? f * wst[(size_t(lane) * G + i) * st + dh + 1] : 0.f;
      for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
      fac[i * 32 + lane] = f;
      if (lane == 0) { hs[2 * i] = M; hs[2 * i + 1] = L; }
    }
    cbar();
    for (int idx = tid; idx < (active ? G * dh : 0); idx += kNC) {
      const int i = idx / dh, d = idx - i * dh;
      float O = 0.f;
#pragma unroll 4
      for (int w = 0; w < kConsumerWarps; ++w) O = fmaf(fac[i * 32 + w], wst[(size_t(w) * G + i) * st + d], O);
      unsigned long long *dst = a.attn_part + (size_t(g * G + i) * a.max_split + split) * st;
      st_tagged(dst + d, O, tag);
      if (d == 0) {
        st_tagged(dst + dh, hs[2 * i], tag);
        st_tagged(dst + dh + 1, hs[2 * i + 1], tag);
      }
    }
    // every split of the group publishes its partial (tagged gl + 1), then
    // each CTA of the group waits for and loads the words it needs into
    // shared memory and merges them (log-sum-exp) into the group's output
    KT(TE_ATTN, 2);
    if (I::ablations && a.grid_sync) {   // the ablation keeps a grid-wide barrier here
      signal(SY_GRID);
      if (!gate(SY_GRID, 0, 0x28, 5)) return;
    }
    // This SM's O projection reads only the merged outputs [r0, r0 + nr) of
    // the group's G*dh: stage every split's (m, l) and those output columns.
    const int r0 = s.misc->sc[ST_O].row0, nr = s.misc->sc[ST_O].nout;
    float *pml = s.vbuf;                       // [G][nsplit][2]
    float *po = pml + 2 * G * kMaxSplit;       // [nsplit][nr]
    bool ok = true;
    for (int q = tid; q < 2 * G * nsplit; q += kNC) {
      const int i = q / (2 * nsplit), r = q - i * 2 * nsplit;
      ok = ok && wait_tagged(a, a.attn_part + (size_t(g * G + i) * a.max_split + (r >> 1)) * st + dh + (r & 1),
                             tag, 0x28, pml[q]);
    }
    for (int q = tid; q < nsplit * nr; q += kNC) {
      const int sp = q / nr, idx = r0 + (q - sp * nr);
      const int i = idx / dh, d = idx - i * dh;
      ok = ok && wait_tagged(a, a.attn_part + (size_t(g * G + i) * a.max_split + sp) * st + d, tag, 0x28, po[q]);
    }
    if (!ok) s.misc->abort = 1;
    cbar();
    if (aborted()) return;
    // log-sum-exp merge of the splits: warp i computes head i's weights
    // exp(m_s - M) / sum_s l_s exp(m_s - M) once (lane = split), then every
    // needed output element is an nsplit-term weighted sum.  The split
    // holding position p is never empty, so the denominator is positive.
    if (warp < G) {
      const int i = warp;
      const float ms = lane < nsplit ? pml[(i * nsplit + lane) * 2] : -INFINITY;
      float M = ms;
      for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float f = ms == -INFINITY ? 0.f : expf(ms - M);
      float L = lane < nsplit ? f * pml[(i * nsplit + lane) * 2 + 1] : 0.f;
      for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
      fac[i * 32 + lane] = f / L;
    }
    cbar();
    float *og = s.svec;   // [G * dh] merged attention output of the group (rows r0.. used)
    for (int q = tid; q < nr; q += kNC) {
      const int idx = r0 + q, i = idx / dh;
      float O = 0.f;
#pragma unroll 4
      for (int sp = 0; sp < nsplit; ++sp) O = fmaf(fac[i * 32 + sp], po[sp * nr + q], O);
      og[idx] = O;
    }
    cbar();
  }

  // ---- column stages (O, down): out[:] += sum_i svals[i] * W_i[:]
  // W_i are the stage's streamed rows (columns of the canonical matrix), svals
  // the matching scalars in shared memory (index = local row).  Each thread
  // owns CPS 4-element output groups and a phase of the tile's rows: rows
  // ph, ph + nseg, ... (8 / CPS of them: a tile holds 8 * nseg / CPS rows).
  // Its words and row scalars of the next tile are loaded before the current
  // tile's arithmetic (one-tile software pipeline across blocks).  At the end
  // of a block, phases are summed in shared memory (nseg > 1) and every group
  // is added to the fp32 accumulator with one vector atomic.
  template <int CPS>
  struct ColWords {
    uint2 w[8 / CPS][CPS];
  };

  template <int CPS>
  __device__ ColWords<CPS> col_words(const StageShape &sh, int ph, int gi, int tpr, int rows) const {
    ColWords<CPS> cw;
    const uint8_t *tile = s.ring + size_t(slot) * kSlotBytes;
#pragma unroll
    for (int q = 0; q < 8 / CPS; ++q) {
      const int r = ph + q * sh.nseg;
      const bool in = r < rows;
      const uint8_t *row = tile + size_t(r) * sh.K * 2;
#pragma unroll
      for (int j = 0; j < CPS; ++j)
        cw.w[q][j] = in ? *reinterpret_cast<const uint2 *>(row + size_t(gi + tpr * j) * 8)
                        : make_uint2(0u, 0u);
    }
    return cw;
  }

  // acc: the accumulator (acc_o or acc_d); parity: the layer's half of it
  __device__ void gemv_cols(int k, const float *svals, float *acc, uint32_t parity) {
    if ((I::cc ? I::cc : a.shape[k].cps) == 1) gemv_cols_impl<1>(k, svals, acc, parity);
    else gemv_cols_impl<2>(k, svals, acc, parity);
  }

  // Accumulates one tile (its rows ph, ph + nseg, ...) into acc2.
  template <int CPS>
  __device__ __forceinline__ void col_tile_math(const ColWords<CPS> &cw, const float *sv, int ph,
                                                int nseg, int rows, float2 (&acc2)[CPS][2]) const {
#pragma unroll
    for (int q = 0; q < 8 / CPS; ++q) {
      const int r = ph + q * nseg;
      const float xv = r < rows ? sv[r] : 0.f;
      const float2 xx = make_float2(xv, xv);
#pragma unroll
      for (int j = 0; j < CPS; ++j) {
        acc2[j][0] = __ffma2_rn(Store<T>::pair(cw.w[q][j].x), xx, acc2[j][0]);
        acc2[j][1] = __ffma2_rn(Store<T>::pair(cw.w[q][j].y), xx, acc2[j][1]);
      }
    }
  }

  template <int CPS>
  __device__ __forceinline__ ColWords<CPS> col_fetch(int k, const StageShape &sh, int ph, int gi,
                                                     int tpr, int rows, uint32_t &sl, bool &ok) {
    ColWords<CPS> cw{};
    sl = slot;
    ok = ok && tile_wait(k);
    if (ok) cw = col_words<CPS>(sh, ph, gi, tpr, rows);
    slot_advance();
    return cw;
  }

  template <int CPS>
  __device__ void gemv_cols_impl(int k, const float *svals, float *acc, uint32_t parity) {
    KP_BEGIN(t_gemv);
    KT(TE_STAGE_BEGIN, k);
    const StageShape sh = a.shape[k];
    const StageCta &c = s.misc->sc[k];
    const int ngrp = sh.K >> 2;                  // 4-element groups of the output
    const int tpr = sh.nseg > 1 ? ngrp : kNC;    // threads per row phase
    const int ph = tid / tpr, gi = tid - ph * tpr;
    const int R = sh.R;
    // A failed wait stops this warp's tile work, but every warp still goes
    // through the same barriers so that none is left waiting.
    bool ok = !aborted();
    for (int bi = 0; bi < c.nblk; ++bi) {
      const Block b = s.misc->blk[c.blk_begin + bi];
      if (b.nrows == 0) continue;
      const int n = (b.nrows + R - 1) / R;
      const int last_rows = b.nrows - (n - 1) * R;
      const float *sv0 = svals + b.lrow0;
      float2 acc2[CPS][2];
#pragma unroll
      for (int j = 0; j < CPS; ++j) acc2[j][0] = acc2[j][1] = make_float2(0.f, 0.f);
      uint32_t sa = 0, sb = 0;
      ColWords<CPS> ca = col_fetch<CPS>(k, sh, ph, gi, tpr, n == 1 ? last_rows : R, sa, ok);
      if (ok) release_slot(sa);
      for (int t = 0; t < n && ok; t += 2) {
        const bool has_b = t + 1 < n;
        const int rows_b = t + 1 < n - 1 ? R : last_rows;
        ColWords<CPS> cb{};
        if (has_b) cb = col_fetch<CPS>(k, sh, ph, gi, tpr, rows_b, sb, ok);
        col_tile_math<CPS>(ca, sv0 + t * R, ph, sh.nseg, t < n - 1 ? R : last_rows, acc2);
        KT(TE_TILE_MATH, 0);
        if (!has_b || !ok) break;
        release_slot(sb);
        KT(TE_TILE_DONE, 0);
        const bool has_a = t + 2 < n;
        if (has_a) ca = col_fetch<CPS>(k, sh, ph, gi, tpr, t + 2 < n - 1 ? R : last_rows, sa, ok);
        col_tile_math<CPS>(cb, sv0 + (t + 1) * R, ph, sh.nseg, rows_b, acc2);
        if (has_a && ok) release_slot(sa);
        KT(TE_TILE_DONE, 0);
      }
      // the block is complete: add its groups into the accumulator
      if (sh.nseg == 1) {
        if (ok) {
#pragma unroll
          for (int j = 0; j < CPS; ++j)
            acc_add4(acc, parity, b.out_off + 4 * (gi + tpr * j),
                     make_float4(acc2[j][0].x, acc2[j][0].y, acc2[j][1].x, acc2[j][1].y));
        }
      } else {
        // several row phases: add them up in shared memory first (CPS == 1)
        float4 *scr = reinterpret_cast<float4 *>(s.vbuf);
        scr[ph * ngrp + gi] = make_float4(acc2[0][0].x, acc2[0][0].y, acc2[0][1].x, acc2[0][1].y);
        cbar();
        if (tid < ngrp && !aborted()) {
          float4 v = scr[tid];
          for (int q = 1; q < sh.nseg; ++q) v = add4(v, scr[q * ngrp + tid]);
          acc_add4(acc, parity, b.out_off + 4 * tid, v);
        }
        cbar();
      }
    }
    if (!ok) s.misc->abort = 1;
    Tbase += c.ntiles;
    cbar();
    KT(TE_STAGE_END, k);
    KP_END(t_gemv, PF_GEMV);
    KP_END(t_gemv, PF_GEMV_K + k);
  }

  // ---- LM head epilogue: logits and the CTA's share of the argmax
  // lm_row() takes each logit as its row block is reduced (thread `row` of the
  // block); lm_fold() then folds the threads' (value, index) pairs into one
  // packed key per step.  bidx starts at a row of this CTA so that the key
  // always names a valid token; a NaN logit never wins a comparison and
  // raises DE_NONFINITE.
  __device__ __forceinline__ void lm_row(int i, float v, float &best, int &bidx) {
    const int row = s.misc->sc[ST_LM].row0 + i;
    if (a.logits_out) a.logits_out[size_t(step - a.logits_step0) * a.vocab + row] = v;
    if (I::sample) a.zbuf[row] = v;
    if (v != v) raise_error(a, DE_NONFINITE | (uint32_t(step & 0xffff) << 8));
    if (v > best || (v == best && row < bidx)) { best = v; bidx = row; }
  }
  __device__ void lm_fold(float best, int bidx) {
    const StageCta &c = s.misc->sc[ST_LM];
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
      atomicMax(a.keys + step, logit_key(best, bidx));
    }
  }

  __device__ __forceinline__ SampleArgs sample_args() const {
    return SampleArgs{a.zbuf,      a.cand, a.psum,        a.keys,     a.uniforms, a.stage_cta, a.sync,
                      a.watchdog_ns, a.sample_t, a.sample_p, a.sample_k, a.vocab,    a.n_ctas};
  }

  __device__ void run() {
    KP_BEGIN(t_total);
    run_body();
    KP_END(t_total, PF_TOTAL);
  }

  __device__ void run_body() {
    const int L = a.n_layers, d = a.d_model;
    const bool lanes = I::lanes && a.n_lanes > 1;
    const int delta = a.lane_delay;
    const uint32_t nc = a.n_ctas;
    const int own_lo = int(int64_t(d) * cta / a.n_ctas);  // residual rows this CTA owns
    const int own_hi = int(int64_t(d) * (cta + 1) / a.n_ctas);
    tok = a.forced ? a.forced[0] : a.first_token;
    for (step = 0; step < a.n_steps; ++step) {
      p = a.pos0 + step;
      // Every CTA sees the same token, so all of them leave together here
      // before an embedding row outside the table could be read.
      if (unsigned(tok) >= unsigned(a.vocab)) {
        raise_error(a, DE_NONFINITE | (uint32_t(step & 0xffff) << 8));
        goto done;
      }
      const bool lm = a.logits_every_step || step == a.n_steps - 1;
#ifdef KIE_PROFILE
      tracing = a.trace && cta == a.trace_cta && step == a.trace_step;
#endif
      for (l = 0; l < L; ++l) {
        gl = uint32_t(step) * L + l;
        KT(TE_LAYER, l & 15);
        const uint32_t cur = gl & 1u, prev = (gl - 1) & 1u;
        // ---------------- RMSNorm + q/k/v rows of the group
        // (every CTA's down contribution to the previous layer is in); the
        // residual entering the layer is staged, its owners keep their rows
        if (gl > 0 && !gate(SY_S2, gl * nc, 0x10, 1)) goto done;
        stage_input([=](int j) { return xin4(j); }, a.gain_attn + size_t(l) * d, d,
                    a.xres + size_t(cur) * d, own_lo, own_hi);
        {
          const StageCta &c = s.misc->sc[ST_QKV];
          // q/k/v rows go out as words tagged gl + 1, which the group's SMs
          // poll directly (the test hook withholds them once, so that the
          // group's waits run out)
          const bool publish = !(a.skip_signal_cta == cta && step == 0 && l == 0);
          auto to_qkv = [&](int i, float v) {
            for (int bi = 0; bi < c.nblk; ++bi) {
              const Block &o = s.misc->blk[c.blk_begin + bi];
              if (unsigned(i - o.lrow0) < unsigned(o.nrows)) {
                if (publish) st_tagged(a.qkv + o.out_off + (i - o.lrow0), v, gl + 1);
                break;
              }
            }
          };
          gemv_rows(ST_QKV, s.vbuf, to_qkv);
        }
        if (aborted()) goto done;
        if (I::ablations && a.grid_sync) signal(SY_GRID);   // the ablation keeps a grid-wide barrier here
        // ---------------- delayed cross-lane sum of the previous layer
        if (lanes && l >= 1) {
          stage_input([=](int j) { return add4(acc4(a.acc_o, prev, j), acc4(a.acc_d, prev, j)); },
                      nullptr, d);
          const StageCta &c = s.misc->sc[ST_MIX];
          float *dst = a.dsum + size_t((l - 1) % delta) * d;
          auto to_dsum = [&](int i, float v) { dst[c.row0 + i] = v; };
          gemv_rows(ST_MIX, s.vbuf, to_dsum);
          if (aborted()) goto done;
        }
        // ---------------- attention of the group, merged in every group CTA
        if (I::ablations && a.grid_sync && !gate(SY_GRID, 0, 0x20, 4)) goto done;
        attention();
        if (aborted()) goto done;
        // ---------------- O projection over the group's attention outputs
        gemv_cols(ST_O, s.svec + s.misc->sc[ST_O].row0, a.acc_o, cur);
        if (aborted()) goto done;
        signal(SY_S1);
        // ---------------- RMSNorm + gate/up + SwiGLU of this CTA's hidden slice
        if (!gate(SY_S1, (gl + 1) * nc, 0x40, 0)) goto done;
        // the previous layer's accumulators were read by every CTA before S1;
        // clear this CTA's rows of them for the layer after next
        if (gl > 0)
          for (int r = own_lo + tid; r < own_hi; r += kNC) {
            a.acc_o[size_t(prev) * d + r] = 0.f;
            a.acc_d[size_t(prev) * d + r] = 0.f;
            if (I::ablations && a.det_sum) {   // the lo sums, 2 d further on
              a.acc_o[size_t(2 + prev) * d + r] = 0.f;
              a.acc_d[size_t(2 + prev) * d + r] = 0.f;
            }
          }
        {
          const float4 *xr = vec4(a.xres, cur);
          stage_input([=](int j) { return add4(__ldcg(xr + j), acc4(a.acc_o, cur, j)); },
                      a.gain_ffn + size_t(l) * d, d);
          float *rs = rsum();
          auto to_rsum = [&](int i, float v) { rs[i] = v; };
          gemv_rows(ST_GU, s.vbuf, to_rsum);
        }
        if (aborted()) goto done;
        {
          const StageCta &c = s.misc->sc[ST_GU];
          const float *rs = rsum();
          float *h = s.svec + kSvecO;
          for (int i = tid; i < c.nout; i += kNC) {
            const float gt = rs[i], up = rs[c.nout + i];
            h[i] = gt / (1.f + expf(-gt)) * up;
          }
          cbar();
        }
        // ---------------- down projection over that slice
        gemv_cols(ST_D, s.svec + kSvecO, a.acc_d, cur);
        if (aborted()) goto done;
        signal(SY_S2);
      }
      if (lm) {
        KT(TE_LAYER, 15);
        ++lm_count;
        const uint32_t last = gl & 1u;   // parity of the last layer
        if (!gate(SY_S2, (gl + 1) * nc, 0x60, 1)) goto done;
        if (lanes) {
          // the last layer's delayed sum, flushed before the final norm
          stage_input([=](int j) { return add4(acc4(a.acc_o, last, j), acc4(a.acc_d, last, j)); },
                      nullptr, d);
          const StageCta &c = s.misc->sc[ST_MIX];
          float *dst = a.dsum + size_t((L - 1) % delta) * d;
          auto to_dsum = [&](int i, float v) { dst[c.row0 + i] = v; };
          gemv_rows(ST_MIX, s.vbuf, to_dsum);
          if (aborted()) goto done;
          signal(SY_MIXF);
          if (!gate(SY_MIXF, lm_count * nc, 0x70, 2)) goto done;
        }
        {
          const float4 *xr = vec4(a.xres, last);
          const int li0 = lanes && L > delta ? L - delta : 0;
          stage_input(
              [=](int j) {
                float4 v = add4(add4(__ldcg(xr + j), acc4(a.acc_o, last, j)), acc4(a.acc_d, last, j));
                if (lanes)
                  for (int li = li0; li < L; ++li)
                    v = add4(v, __ldcg(reinterpret_cast<const float4 *>(a.dsum + size_t(li % delta) * d) + j));
                return v;
              },
              a.gain_final, d);
          float best = -INFINITY;
          int bidx = s.misc->sc[ST_LM].row0;
          auto to_lm = [&](int i, float v) { lm_row(i, v, best, bidx); };
          gemv_rows(ST_LM, s.vbuf, to_lm);
          if (aborted()) goto done;
          lm_fold(best, bidx);
          if constexpr (I::sample) {
            if (a.sample_k > 0) local_topk(sample_args(), s, tid, cta);
          }
        }
        signal(SY_TOK);
        if (!gate(SY_TOK, lm_count * nc, 0x80, 3)) goto done;
        int next;
        if constexpr (I::sample) {
          next = a.sample_k > 0 ? sample_topk(sample_args(), s, tid, step)
                                : sample_full(sample_args(), s, tid, cta, step, lm_count);
          if (next < 0) goto done;
        } else {
          next = key_row(__ldcg(a.keys + step));
        }
        if (cta == 0 && tid == 0) a.out_tokens[step] = next;
        tok = next;
      }
      if (a.forced && step + 1 < a.n_steps) tok = a.forced[step + 1];
    }
  done:
    return;
  }
};

template <typename T, int V, int GS, int DHS, int CQ, int CR, int CC, int CM>
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
  s.svec = s.part + a.part_floats;
  s.misc = reinterpret_cast<Misc *>(s.svec + kSvecFloats);

  for (int i = tid; i < a.part_floats; i += kThreads) s.part[i] = 0.f;   // row sums start at zero
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
    for (int i = 0; i < kConsumerWarps; ++i) s.misc->wwait[i] = 0;
    s.misc->tn = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (tid >= kNC) {
    if (tid == kNC) {
#ifdef KIE_PROFILE
      const long long t0 = clock64();
#endif
      Producer<V> pr(a, s, cta);
      pr.run();
#ifdef KIE_PROFILE
      s.misc->prof[PF_PROD_TOTAL] += clock64() - t0;
      s.misc->prof[PF_TILES] = pr.T;
#endif
    }
    __syncwarp();
  } else {
    Consumer<T, V, GS, DHS, CQ, CR, CC, CM> c(a, s, tid, cta);
    c.run();
    // a CTA that gave up makes every other CTA (and its own producer) leave
    if (tid == 0 && c.aborted()) atomicExch(sync_at(a, SY_ABORT), 1u);
  }
  __syncthreads();
#ifdef KIE_PROFILE
  if (tid == 0) {
    long long sum = 0, mx = 0, mn = s.misc->wwait[0];
    for (int w = 0; w < kConsumerWarps; ++w) {
      sum += s.misc->wwait[w];
      mx = max(mx, s.misc->wwait[w]);
      mn = min(mn, s.misc->wwait[w]);
    }
    s.misc->prof[PF_WAIT_ALL] = sum / kConsumerWarps;
    s.misc->prof[PF_WAIT_ALL + 1] = mx;
    s.misc->prof[PF_WAIT_ALL + 2] = mn;
  }
  __syncthreads();
  if (a.prof && tid < kProfSlots) a.prof[size_t(cta) * kProfSlots + tid] = s.misc->prof[tid];
  if (a.trace && cta == a.trace_cta && tid == 0) a.trace[0] = uint32_t(s.misc->tn);
#endif
}

// ------------------------------------------------------------------ weight repack
// Builds the per-SM weight streams from the canonical weights.  A plain job
// copies nrows canonical rows as they are; a transposed job writes nrows
// columns of a row-major [K, src_ld] matrix as rows of K elements (through a
// 32 x 32 shared-memory tile so that both sides stay coalesced).
__global__ void __launch_bounds__(256) repack_kernel(const uint16_t *__restrict__ src,
                                                     uint8_t *__restrict__ dst,
                                                     const RepackJob *__restrict__ jobs, int njobs) {
  __shared__ uint16_t tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int jb = blockIdx.x; jb < njobs; jb += gridDim.x) {
    const RepackJob job = jobs[jb];
    uint16_t *out = reinterpret_cast<uint16_t *>(dst + job.dst_byte);
    const uint16_t *in = src + job.src_elem;
    if (job.trans == 2) {
      // rows of a row block's column tiles, 16-byte chunks swizzled by tile row
      const int nchunk = job.K >> 3, cpt = job.kb >> 3;
      const int64_t nvec = int64_t(job.nrows) * nchunk;
      for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
        const int i = int(v / nchunk), q = int(v - int64_t(i) * nchunk);
        const int t = q / cpt, c = q - t * cpt, r = job.rb0 + i;
        const int64_t e = (int64_t(t) * job.rb + r) * job.kb + int64_t(c ^ (r & 7)) * 8;
        reinterpret_cast<uint4 *>(out)[e >> 3] = *reinterpret_cast<const uint4 *>(in + int64_t(i) * job.K + q * 8);
      }
      continue;
    }
    if (!job.trans) {
      const int64_t nvec = int64_t(job.nrows) * job.K / 8;
      for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x)
        reinterpret_cast<uint4 *>(out)[v] = *reinterpret_cast<const uint4 *>(in + v * 8);
      continue;
    }
    const int ncol = job.nrows, K = job.K;
    for (int r0 = 0; r0 < K; r0 += 32)
      for (int c0 = 0; c0 < ncol; c0 += 32) {
        for (int rr = ty; rr < 32; rr += 8) {
          const int r = r0 + rr, cc = c0 + tx;
          tile[rr][tx] = (r < K && cc < ncol) ? in[int64_t(r) * job.src_ld + cc] : uint16_t(0);
        }
        __syncthreads();
        for (int ii = ty; ii < 32; ii += 8) {
          const int cc = c0 + ii, r = r0 + tx;
          if (cc < ncol && r < K) out[int64_t(cc) * K + r] = tile[tx][ii];
        }
        __syncthreads();
      }
  }
}

// ------------------------------------------------------------------ host entry points
size_t monokernel_smem_bytes(int ring_slots, int vbuf_floats, int part_floats) {
  return size_t(ring_slots) * kSlotBytes + size_t(ring_slots) * 16 +
         size_t(vbuf_floats + part_floats + kSvecFloats) * 4 + sizeof(Misc);
}

int monokernel_threads() { return kThreads; }

bool monokernel_profiled() {
#ifdef KIE_PROFILE
  return true;
#else
  return false;
#endif
}

// variant: KV_GENERAL, KV_SAMPLE and KV_LANES bits (see "kernel instances").
// The dense variants, greedy and sampling, come specialised for the shapes of the
// 2.3B-class models (G 2, dh 128, widths q/k/v 4, rows 1, columns 1) and of
// the 8B-class one (G 4, dh 128, widths 2, 1, 2), other shapes running the
// runtime-shape instance; the lanes variant exists for the lane-structured
// model's shape (G 1, dh 128, widths 2, 1, 1, lane mix 4), other lane
// models running the general instance.
template <typename T>
static const void *pick(int variant, const InstShape &k) {
  if (k.G == 2 && k.dh == 128 && k.cq == 4 && k.cr == 1 && k.cc == 1) {
    if (variant == 0) return reinterpret_cast<const void *>(&monokernel<T, 0, 2, 128, 4, 1, 1, 0>);
    if (variant == KV_SAMPLE)
      return reinterpret_cast<const void *>(&monokernel<T, KV_SAMPLE, 2, 128, 4, 1, 1, 0>);
  }
  if (k.G == 4 && k.dh == 128 && k.cq == 2 && k.cr == 1 && k.cc == 2) {
    if (variant == 0) return reinterpret_cast<const void *>(&monokernel<T, 0, 4, 128, 2, 1, 2, 0>);
    if (variant == KV_SAMPLE)
      return reinterpret_cast<const void *>(&monokernel<T, KV_SAMPLE, 4, 128, 2, 1, 2, 0>);
  }
  if (variant == KV_LANES) {
    if (k.G == 1 && k.dh == 128 && k.cq == 2 && k.cr == 1 && k.cc == 1 && k.cm == 4)
      return reinterpret_cast<const void *>(&monokernel<T, KV_LANES, 1, 128, 2, 1, 1, 4>);
    variant = KV_GENERAL;
  }
  switch (variant & 3) {
    case 0: return reinterpret_cast<const void *>(&monokernel<T, 0, 0, 0, 0, 0, 0, 0>);
    case 1: return reinterpret_cast<const void *>(&monokernel<T, 1, 0, 0, 0, 0, 0, 0>);
    case 2: return reinterpret_cast<const void *>(&monokernel<T, 2, 0, 0, 0, 0, 0, 0>);
    default: return reinterpret_cast<const void *>(&monokernel<T, 3, 0, 0, 0, 0, 0, 0>);
  }
}
const void *monokernel_fn(int dtype, int variant, const InstShape &shape) {
  return dtype == 0 ? pick<__half>(variant, shape) : pick<__nv_bfloat16>(variant, shape);
}

cudaError_t launch_repack(const uint16_t *src, uint8_t *dst, const RepackJob *jobs, int njobs,
                          cudaStream_t st) {
  if (njobs == 0) return cudaSuccess;
  repack_kernel<<<min(njobs, 4096), 256, 0, st>>>(src, dst, jobs, njobs);
  return cudaGetLastError();
}

}  // namespace kie
