// Internal structures shared by the host side (kie_api.cu) and the persistent
// decode kernel (monokernel.cu).  Not part of the public ABI.
#pragma once
#include <stdint.h>
#include <vector_types.h>

namespace kie {

// Stage kinds of one decode step, in the order a layer runs them.
enum StageKind : int {
  ST_QKV = 0,  // RMSNorm(attn) + fused q/k/v GEMV            -> qkv
  ST_O = 1,    // O GEMV + residual add                        -> x (and u)
  ST_GU = 2,   // RMSNorm(ffn) + gate/up GEMV + SwiGLU         -> h
  ST_D = 3,    // down GEMV + residual add                     -> x (and u)
  ST_MIX = 4,  // lane models: delayed cross-lane sum M_i u_i  -> dsum[i % delta]
  ST_LM = 5,   // final RMSNorm + LM head GEMV + argmax        -> logits / token
  ST_COUNT = 6
};

// Global counters used as epoch barriers (one 128-byte line each).
enum SyncSlot : int {
  SY_QKV = 0,    // CTAs that finished the QKV stage
  SY_OREADY = 1, // KV-head groups whose attention output is merged
  SY_X1 = 2,     // CTAs that finished the O stage
  SY_H = 3,      // CTAs that finished the gate/up stage
  SY_X2 = 4,     // CTAs that finished the down stage
  SY_MIXF = 5,   // CTAs that finished the final delayed-sum flush
  SY_TOK = 6,    // CTAs that folded their LM-head rows into the argmax
  SY_ABORT = 7,  // nonzero: a CTA gave up; everyone leaves
  SY_STATUS = 8, // first device error code (0 = none)
  SY_ATTN0 = 16, // per KV-head attention split counters start here
};
constexpr int kSyncStride = 32;  // uint32 words per counter (128 bytes)

// Per-stage constants shared by every CTA.  A tile is R whole rows (at most
// kSlotBytes).  All consumer warps share every tile: warp w takes row group
// w / nseg (rpw consecutive rows) and column split w % nseg (cps 8-element
// chunks of each of those rows), so each lane holds at most 4 chunks.
struct StageShape {
  int32_t K;       // reduction length of every row
  int32_t R;       // rows per tile (power of two)
  int32_t nseg;    // column splits per row = partial sums per row
  int32_t rpw;     // rows per warp (1 unless R > 16)
  int32_t cps;     // 8-element chunks per (row, split) = K / 8 / nseg
  int32_t in_len;  // length of the stage input vector
  int32_t out_len; // length of the stage output vector
};

// One CTA's share of a stage: output rows [row0, row0 + nout).
struct StageCta {
  int32_t row0, nout;
  int32_t nlocal;     // local rows held in partial sums (2*nout for gate/up)
  int32_t ntiles;
  int32_t blk_begin;  // first block, counted from the CTA's own first block
  int32_t nblk;
  int64_t bytes;      // stream bytes of one instance of this stage
};

// A run of rows of one CTA's stage that read the same input slice.
struct Block {
  int32_t lrow0;   // first local row
  int32_t nrows;
  int32_t in_off;  // offset of the rows' input within the stage input vector
  int32_t tile0;   // index of the block's first tile within the stage
};

// Copy job of the weight repack: one block of one stage instance.
struct RepackJob {
  int64_t src_elem;  // canonical element offset of the block's first row
  int64_t dst_byte;  // byte offset in the streaming buffer
  int32_t nrows, K, KT, R;
};

// Per-SM activity counters of the profiling build (SM clock cycles).
enum ProfSlot : int {
  PF_TOTAL = 0,       // consumer thread 0: whole launch
  PF_GATE = 1,        // waiting for other SMs (epoch counters)
  PF_GEMV = 2,        // GEMV stages except the LM head (incl. ring waits)
  PF_FULLWAIT = 3,    // warp 0: waiting for weight tiles to land (ring empty)
  PF_ATTN = 4,        // attention (incl. the merge)
  PF_STAGE = 5,       // input staging and RMSNorm
  PF_SIGNAL = 6,      // end-of-stage barrier + release
  PF_LM = 7,          // LM-head GEMV
  PF_PROD_EMPTY = 8,  // (unused: the copy pump never blocks)
  PF_PROD_TOTAL = 9,  // (unused)
  PF_TILES = 10,      // weight tiles issued
  PF_NGATE = 11,      // number of dependency waits
  PF_GEMV_K = 12,     // 12..17: GEMV time per stage kind
  PF_GATE_K = 18,     // 18..24: dependency-wait time per counter (SyncSlot order)
};
constexpr int kProfSlots = 32;

constexpr int kMaxBlocksPerCta = 64;
constexpr int kSlotBytes = 32768;  // one bulk copy per tile: >= 16 KB keeps HBM saturated
constexpr int kConsumerWarps = 16;

struct KernelArgs {
  // model
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  int32_t n_lanes, lane_delay;
  int32_t lane_width, lane_heads, lane_kv_heads, lane_ffn;
  float rms_eps, attn_scale;
  int32_t max_seq;
  // plan
  int32_t n_ctas, ring_slots, vbuf_floats, part_floats;
  StageShape shape[ST_COUNT];
  const StageCta *stage_cta;  // [ST_COUNT][n_ctas]
  const Block *blocks;
  const int32_t *cta_blk_begin;   // [n_ctas + 1] first block of each CTA in `blocks`
  const int64_t *cta_stream_off;  // [n_ctas] byte offset of each CTA's stream
  const uint8_t *wstream;
  // weights outside the stream
  const uint16_t *embed;     // [V, d] storage bits
  const float *gain_attn;    // [L, d] fp32
  const float *gain_ffn;     // [L, d]
  const float *gain_final;   // [d]
  const float2 *rope_cs;     // [max_seq, dh/2] (cos, sin)
  // state
  uint16_t *kcache, *vcache; // [L, Hkv, max_seq, dh]
  float *x;      // [d] residual
  float *qkv;    // [(Hq + 2 Hkv) dh]
  float *attn_o; // [Hq dh]
  float *hbuf;   // [F]
  float *ubuf;   // [2, d] lane outputs of the last two layers
  float *dsum;   // [delta, d] delayed cross-lane sums
  float *attn_part;  // [Hq, max_split, dh + 2] per-split attention partials
  int32_t max_split; // most CTAs sharing one KV head
  uint32_t *sync;
  unsigned long long *keys;  // [n_steps] packed argmax keys (zeroed by host)
  // run
  int32_t pos0, n_steps;
  int32_t first_token;          // token fed at step 0 when forced == nullptr
  const int32_t *forced;        // device [n_steps] or nullptr
  int32_t logits_every_step;    // 1: LM head every step; 0: only at the last step
  int32_t *out_tokens;          // device [n_steps]
  float *logits_out;            // device [n_steps, V] or nullptr
  uint64_t watchdog_ns;
  int32_t skip_signal_cta;      // test hook, -1 = off
  int32_t l2_prefetch_tiles;    // tiles the producer pulls into L2 beyond the ring
  unsigned long long *prof;     // [n_ctas][kProfSlots] (profiling build), or nullptr
};

}  // namespace kie
