// Internal structures shared by the host side (kie_api.cu) and the persistent
// decode kernel (monokernel.cu).  Not part of the public ABI.
#pragma once
#include <stdint.h>
#include <vector_types.h>

namespace kie {

// Stage kinds of one decode step, in the order a layer streams them.
enum StageKind : int {
  ST_QKV = 0,  // RMSNorm(attn) + q/k/v rows of this CTA's KV-head group   -> qkv
  ST_O = 1,    // O projection split along its input: the Wo columns of the
               // attention outputs this CTA holds                          -> acc_o (atomics)
  ST_GU = 2,   // RMSNorm(ffn) + gate/up rows of this CTA's hidden slice + SwiGLU -> h (smem)
  ST_D = 3,    // down projection split along its input: Wd columns of that slice -> acc_d
  ST_MIX = 4,  // lane models: delayed cross-lane sum M_i u_i (rows)        -> dsum[i % delta]
  ST_LM = 5,   // final RMSNorm + LM head rows + argmax                     -> logits / token
  ST_COUNT = 6
};

// Global counters used as epoch barriers (one 128-byte line each).
enum SyncSlot : int {
  SY_S1 = 0,     // CTAs whose O contribution is in acc_o
  SY_S2 = 1,     // CTAs whose down contribution is in acc_d
  SY_MIXF = 2,   // CTAs that finished the final delayed-sum flush
  SY_TOK = 3,    // CTAs that folded their LM-head rows into the argmax
  SY_ABORT = 4,  // nonzero: a CTA gave up; everyone leaves
  SY_STATUS = 5, // first device error code (0 = none)
  SY_GRID = 6,   // grid-barrier mode: signals made by all CTAs together
  SY_COUNT = 8,  // counters in all (the KV group's q/k/v and attention partials are
                 // exchanged as tagged words, without counters)
};
constexpr int kSyncStride = 32;  // uint32 words per counter (128 bytes)

// Per-SM activity counters of the profiling build (SM clock cycles).
enum ProfSlot : int {
  PF_TOTAL = 0,       // consumer thread 0: whole launch
  PF_GATE = 1,        // waiting for other SMs (epoch counters)
  PF_GEMV = 2,        // weight stages except the LM head (incl. ring waits)
  PF_FULLWAIT = 3,    // warp 0: waiting for weight tiles to land (ring empty)
  PF_ATTN = 4,        // attention and the merge of the group's partials
  PF_STAGE = 5,       // input staging and RMSNorm
  PF_SIGNAL = 6,      // end-of-stage barrier + release
  PF_LM = 7,          // LM-head GEMV
  PF_PROD_EMPTY = 8,  // producer: waiting for a free slot (ring full)
  PF_PROD_TOTAL = 9,  // producer: whole launch
  PF_TILES = 10,      // weight tiles issued
  PF_NGATE = 11,      // number of dependency waits
  PF_GEMV_K = 12,     // 12..17: time per stage kind
  PF_GATE_K = 18,     // 18..23: waiting time on S1, S2, MIXF, TOK, q/k/v group, attention group
  PF_WAIT_ALL = 24,   // 24..26: tile waits per consumer warp: mean, max, min over warps
};
constexpr int kProfSlots = 32;

// Event types of the profiling build's trace (4 bits) -- the argument (4 bits)
// is a stage kind, a wait kind or a sub-step.
enum TraceEvent : int {
  TE_LAYER = 0,        // a layer begins (argument: layer & 15; 15 = LM head)
  TE_GATE_BEGIN = 1,   // waiting for other SMs (argument: counter kind)
  TE_GATE_END = 2,
  TE_SIGNAL_BEGIN = 3, // end-of-stage barrier, then the release
  TE_SIGNAL_END = 4,
  TE_NORM_BEGIN = 5,
  TE_NORM_END = 6,
  TE_STAGE_BEGIN = 7,  // a weight stage (argument: stage kind)
  TE_STAGE_END = 8,
  TE_TILE_WAIT = 9,    // warp 0 starts waiting for a tile
  TE_TILE_READY = 10,
  TE_TILE_DONE = 11,   // warp 0 released the tile
  TE_ATTN = 12,        // attention: 0 begin, 1 positions folded, 2 partials written, 3 merged
  TE_TILE_LOADED = 13, // warp 0 has the tile's words in registers (row stages)
  TE_TILE_MATH = 14,   // warp 0 finished the tile's arithmetic
};
constexpr int kTraceCap = 1 << 16;

// Per-stage constants shared by every CTA.
//  Row stages (QKV, GU, MIX, LM): out[row] = sum_k W[row][k] in[k].  A CTA's
//    rows of the stage are cut into row blocks of at most R = 128 / cps rows
//    that share one input slice; a row block streams as K / (128 cps) tiles,
//    tile t holding columns [t 128 cps, (t+1) 128 cps) of every row of the
//    block (rows * 256 cps bytes, at most kSlotBytes), row-major, with the
//    16-byte chunk c of row r stored at chunk position c ^ (r & 7).  Lane l
//    of every consumer warp owns rows l, l + 32, ... of the block; warp w
//    owns chunks [w cps, (w+1) cps) of each tile, so it accumulates its
//    rows' partial dot products in registers over the block's tiles, and the
//    16 warps' partials are added in a fixed order once per row block.
//  Column stages (O, D): out[:] += sum_row s[row] W[row][:], where a row is
//    a column of the canonical matrix; a tile is R whole rows.  Thread t takes
//    row phase t / ngrp and 4-element output groups t % ngrp + ngrp * j
//    (j < cps); nseg phases.
struct StageShape {
  int32_t K;       // row length (row stages: reduction length; column stages: output length)
  int32_t R;       // row stages: most rows of a row block; column stages: rows per tile
  int32_t nseg;    // column stages: row phases (row stages: 1)
  int32_t norm;    // row stages: width of the RMSNorm slices of the input (0: no norm)
  int32_t cps;     // row stages: 16-byte chunks per lane per row of a tile (1, 2, 4);
                   // column stages: 4-element output groups per thread
  int32_t in_len;  // length of the stage input vector
  int32_t out_len; // length of the stage output vector
  int32_t cols;    // 1 for column stages
};

// One CTA's share of a stage.
struct StageCta {
  int32_t row0, nout; // GU: hidden slice [row0, row0 + nout); MIX, LM: output rows
  int32_t nlocal;     // local rows (row sums of row stages, scalars of column stages)
  int32_t ntiles;
  int32_t blk_begin;  // first output block, counted from the CTA's own first block
  int32_t nblk;
  int64_t bytes;      // stream bytes of one instance of this stage
  int32_t rb_begin;   // row stages: first row block (same numbering as blk_begin)
  int32_t nrb;        // row stages: row blocks
};

// A run of rows of one CTA's stage.  Output blocks (blk_begin): rows with one
// output place (and, for row stages, one input slice).  Row blocks of row
// stages (rb_begin): the units the GEMV tiles, at most StageShape::R rows of
// one input slice.
struct Block {
  int32_t lrow0;   // first local row
  int32_t nrows;
  int32_t in_off;  // row stages: offset of the rows' input in the stage input vector
  int32_t tile0;   // index of the block's first tile within the stage
  int32_t out_off; // output blocks of row stages: output index of the first row; column
                   // stages: offset of the block's output slice in the d-vector
  int32_t pad;
};

// Copy job of the weight repack: one block of one stage instance.
//  trans == 0: nrows canonical rows of K elements, copied as they are;
//  trans == 1: nrows columns of a row-major matrix with K rows and row stride
//              src_ld, each written as one row of K elements;
//  trans == 2: nrows canonical rows of K elements (consecutive rows of one
//              matrix), rows rb0 .. rb0 + nrows - 1 of a row block of rb rows
//              whose tiles of kb columns start at dst_byte; chunk c (8
//              elements) of tile row r goes to chunk position c ^ (r & 7).
struct RepackJob {
  int64_t src_elem;  // canonical element offset of the first row (or first column's top)
  int64_t dst_byte;  // byte offset in the streaming buffer
  int32_t nrows, K, trans, src_ld;
  int32_t rb, rb0, kb, pad;
};

constexpr int kMaxBlocksPerCta = 64;
constexpr int kSlotBytes = 32768;  // one bulk copy per tile: >= 16 KB keeps HBM saturated
constexpr int kConsumerWarps = 16;
constexpr int kMaxLocal = 256;     // scalars a column stage holds per CTA
constexpr int kMaxRowBlock = 128;  // rows of a row block (lane l: rows l + 32 j, j < 4)
constexpr int kPartialFloats = 2 * kConsumerWarps * kMaxRowBlock;  // double-buffered warp partials
constexpr int kMaxRowSums = 1024;  // row sums a non-LM row stage keeps per CTA
constexpr int kMaxSplit = 32;      // CTAs that share one KV head's positions (others only merge)
constexpr int kMaxTopK = 64;       // largest top-k of the sampler (candidates kept per CTA)
constexpr int kMaxSampleRows = 2048;  // LM-head rows per CTA that a top-k cut can sort in shared memory

// What a kernel instance may fix at compile time (see monokernel.cu, "kernel
// instances"): attention shape and GEMV tile widths; a launch compares the
// model's and its plan's values with an instance's before using it.
struct InstShape {
  int32_t G, dh;   // query heads per KV head, head size
  int32_t cq, cr;  // row-stage widths (cps): q/k/v; gate/up and LM head (0: they differ)
  int32_t cc;      // column-stage width (cps) of O and down (0: they differ)
  int32_t cm;      // lane models: row-stage width of the lane mix (0: dense)
};

struct KernelArgs {
  // model
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  int32_t n_lanes, lane_delay;
  int32_t lane_width, lane_heads, lane_kv_heads, lane_ffn;
  float rms_eps, attn_scale;
  int32_t max_seq;
  // plan
  int32_t n_ctas, ring_slots, vbuf_floats, part_floats;
  int32_t rsum_off;             // row sums of the last row stage start here in `part`
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
  float *xres;   // [2, d] residual entering global layer G, in xres[G % 2] (row owners write it)
  float *acc_o;  // [2, d] attention sublayer output of layer G (atomic sums; zero when reused);
                 // in deterministic mode followed by [2, d] sums of the lo parts
  float *acc_d;  // [2, d] MLP sublayer output of layer G (same storage as acc_o)
  unsigned long long *qkv;  // [(Hq + 2 Hkv) dh] this step's q/k/v, tagged words (layer + 1)
  float *dsum;   // [delta, d] delayed cross-lane sums
  unsigned long long *attn_part;  // [Hq, max_split, dh + 2] per-split attention partials, tagged
  int32_t max_split; // most CTAs sharing one KV head
  uint32_t *sync;
  unsigned long long *keys;  // [n_steps] packed argmax keys (zeroed by host)
  // run
  int32_t pos0, n_steps;
  int32_t first_token;          // token fed at step 0 when forced == nullptr
  const int32_t *forced;        // device [n_steps] or nullptr
  int32_t logits_every_step;    // 1: LM head every step; 0: only at the last step
  int32_t *out_tokens;          // device [n_steps]
  float *logits_out;            // device [n_steps, V] or nullptr; step s writes row s - logits_step0
  int32_t logits_step0;
  // sampling at the LM head (greedy argmax when sample_t == 0)
  float sample_t;               // temperature
  int32_t sample_k;             // top-k: 0 = no cut (sample_p is then 1), else 1 .. kMaxTopK
  float sample_p;               // top-p within the top-k tokens, in (0, 1]
  const float *uniforms;        // device [n_steps]: each step's uniform in [0, 1)
  float *zbuf;                  // device [V]: the step's logits
  unsigned long long *cand;     // device [n_ctas][kMaxTopK]: each CTA's largest logit keys
  unsigned long long *psum;     // device [n_ctas]: tagged per-CTA probability sums (no top-k cut)
  uint64_t watchdog_ns;
  int32_t skip_signal_cta;      // test hook, -1 = off
  int32_t grid_sync;            // 1: every dependency wait is a grid-wide barrier
  int32_t det_sum;              // 1: O / down sums split into exact hi / lo fp32 sums (order-independent)
  int32_t l2pf_tiles;           // L2 look-ahead while the ring is full: most tiles (0 = off)
  int32_t l2pf_delay;           //   SM cycles of waiting for a free slot before it starts
  int32_t l2pf_pace;            //   SM cycles between two look-ahead requests
  unsigned long long *prof;     // [n_ctas][kProfSlots] (profiling build), or nullptr
  unsigned long long *trace;    // [1 + trace_cap] event trace (profiling build), or nullptr
  int32_t trace_cap, trace_cta, trace_step;
};

}  // namespace kie
