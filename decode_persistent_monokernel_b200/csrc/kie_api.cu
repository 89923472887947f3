// Host side of libkie.so: the C ABI declared in include/kie.h.
//
// kie_create plans how the decode step's weight rows are split over the SMs,
// copies the canonical weights into one contiguous stream per SM in the order
// that SM consumes them (the per-SM weight stream the persistent kernel's
// producer warp reads with bulk copies), and allocates the KV cache and
// activation buffers.  kie_prefill / kie_decode launch the persistent kernel
// once per call, cooperatively, with one CTA per SM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/kie.h"
#include "kie_internal.h"
#include "prefill_internal.h"

namespace kie {
size_t monokernel_smem_bytes(int ring_slots, int vbuf_floats, int part_floats);
int monokernel_threads();
bool monokernel_profiled();
// variant bits: 1 = the general instance (lane models, grid-barrier and
// exact-sum ablations, L2 look-ahead), 2 = the sampler compiled in, 4 = the
// lanes instance (lane models without ablations); shape:
// the model's attention shape and its plan's GEMV widths, for which the dense
// greedy instance may be specialised
const void *monokernel_fn(int dtype, int variant, const InstShape &shape);
cudaError_t launch_repack(const uint16_t *src, uint8_t *dst, const RepackJob *jobs, int njobs,
                          cudaStream_t st);
}  // namespace kie

using namespace kie;

static thread_local std::string g_last_error;

static void set_error(const char *what, cudaError_t e) {
  char buf[512];
  snprintf(buf, sizeof buf, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
  g_last_error = buf;
}

// ---------------------------------------------------------------- canonical layout
namespace {

// Rows of one stage's per-CTA row space that come from one canonical matrix.
struct Piece {
  int64_t src;      // canonical element offset (layer 0) of the first row, or of
                    // the first column's top element for transposed pieces
  int64_t src2;     // second source (up rows of a gate/up piece), or -1
  int32_t rows, K, in_off, out_off;
  int32_t trans, ld;  // transposed pieces: rows are columns of a [K, ld] matrix
};

struct Layout {
  int64_t embed, final_norm, lm_head, total;
  int64_t layer0, layer_stride, lane_stride;
  // offsets inside one lane of layer 0 (relative to the lane's start)
  int64_t attn_norm, wq, wk, wv, wo, ffn_norm, wg, wu, wd;
  int64_t mix;  // relative to the layer start (lane models)
};

Layout make_layout(const kie_model_desc &m) {
  Layout L{};
  const int64_t d = m.d_model, V = m.vocab, dh = m.head_dim;
  const int64_t nl = m.n_lanes, dl = d / nl, hq = m.n_heads / nl, hkv = m.n_kv_heads / nl,
                fl = m.ffn_dim / nl;
  int64_t o = 0;
  L.embed = o; o += V * d;
  L.layer0 = o;
  int64_t q = 0;
  L.attn_norm = q; q += dl;
  L.wq = q; q += hq * dh * dl;
  L.wk = q; q += hkv * dh * dl;
  L.wv = q; q += hkv * dh * dl;
  L.wo = q; q += dl * hq * dh;
  L.ffn_norm = q; q += dl;
  L.wg = q; q += fl * dl;
  L.wu = q; q += fl * dl;
  L.wd = q; q += dl * fl;
  L.lane_stride = q;
  L.mix = nl * q;
  L.layer_stride = nl * q + (nl > 1 ? d * d : 0);
  o += m.n_layers * L.layer_stride;
  L.final_norm = o; o += d;
  L.lm_head = o; o += V * d;
  L.total = o;
  return L;
}

struct Plan {
  int n_ctas = 0;
  StageShape shape[ST_COUNT]{};
  std::vector<StageCta> stage_cta;   // [ST_COUNT][n_ctas]
  std::vector<Block> blocks;
  std::vector<int32_t> cta_blk_begin;
  std::vector<int64_t> cta_stream_off;
  std::vector<RepackJob> jobs;
  int64_t stream_bytes = 0;
  int vbuf_floats = 0, part_floats = 0, ring_slots = 0;
  int rsum_off = 0;          // start of the row sums inside the partials buffer
  size_t smem = 0;
  int max_split = 0;
  int64_t weight_bytes_per_step = 0;
};

// Row stage whose rows have K elements (see StageShape); the chunk width cps
// and the row-block size R are set once the plan knows the stage's runs.
const char *make_shape(int K, int in_len, int out_len, int norm, StageShape &s) {
  s = StageShape{};
  s.K = K;
  s.in_len = in_len;
  s.out_len = out_len;
  s.norm = norm;
  // a tile spans 128 cps columns (16 warps x cps 16-byte chunks), so K must
  // be a multiple of 128; K / 128 a power of two keeps every cps choice exact
  if (K % 128 || K < 128 || K > 4096 || ((K >> 7) & ((K >> 7) - 1)))
    return "row length must be 128 times a power of two, at most 4096";
  s.nseg = 1;
  s.cps = 1;
  s.R = kMaxRowBlock;
  return nullptr;
}

// Chunk width of a row stage whose longest run of rows with one input slice
// (on any CTA) has `run` rows: the widest tile (most columns) whose row blocks
// still hold such a run whole, within 4 chunks per lane and K.
void set_row_tiling(StageShape &s, int run) {
  int c = run <= 32 ? 4 : run <= 64 ? 2 : 1;
  while (c > 1 && 128 * c > s.K) c >>= 1;
  s.cps = c;
  s.R = kMaxRowBlock / c;
}

// Tile shape of a column stage whose rows (canonical columns) have n_out
// elements: the output vector length.
const char *make_cshape(int n_out, int in_len, StageShape &s) {
  s = StageShape{};
  s.cols = 1;
  s.K = n_out;
  s.in_len = in_len;
  s.out_len = n_out;
  const int nthreads = kConsumerWarps * 32;
  const int ngrp = n_out / 4;
  if (n_out % 4 || 2 * n_out > kSlotBytes) return "output slice of a split projection must fit one slot";
  if (ngrp >= nthreads) {
    if (ngrp % nthreads) return "split projection output must be a multiple of 2048 or divide it";
    s.cps = ngrp / nthreads;
    s.nseg = 1;
  } else {
    if (nthreads % ngrp) return "split projection output must be a multiple of 2048 or divide it";
    s.cps = 1;
    s.nseg = nthreads / ngrp;
  }
  if (s.cps > 4) return "split projection output too long";
  int R = 1;
  while (R * 2 * 2 * n_out <= kSlotBytes && R < 64) R *= 2;
  s.R = R;
  if ((R + s.nseg - 1) / s.nseg > 8) return "split projection tile has more than 8 rows per thread";
  return nullptr;
}

// Blocks of one CTA's row range [r0, r1) of a stage; `up` selects the second
// source of gate/up pieces.  Returns the layer-0 source of each block.
void cut_blocks(const std::vector<Piece> &pieces, int r0, int r1, bool up, int lrow_base,
                const StageShape &sh, int &tile, std::vector<Block> &blk,
                std::vector<Piece> &src) {
  int base = 0;
  for (const Piece &pc : pieces) {
    const int a = std::max(r0, base), b = std::min(r1, base + pc.rows);
    if (a < b) {
      Block B{};
      B.lrow0 = lrow_base + (a - r0);
      B.nrows = b - a;
      B.in_off = pc.in_off;
      B.tile0 = tile;
      B.out_off = pc.trans ? pc.out_off : pc.out_off + (a - base);
      if (sh.cols) tile += (B.nrows + sh.R - 1) / sh.R;
      blk.push_back(B);
      Piece one = pc;
      one.rows = b - a;
      const int64_t s0 = up ? pc.src2 : pc.src;
      one.src = pc.trans ? s0 + (a - base) : s0 + int64_t(a - base) * pc.K;
      src.push_back(one);
    }
    base += pc.rows;
  }
}

// Runs of consecutive output blocks with one input slice (a row stage's local
// rows are in block order).
std::vector<std::pair<int, int>> input_runs(const std::vector<Block> &blk) {
  std::vector<std::pair<int, int>> runs;   // (first local row, rows)
  for (size_t i = 0; i < blk.size();) {
    size_t j = i + 1;
    int n = blk[i].nrows;
    while (j < blk.size() && blk[j].in_off == blk[i].in_off && blk[j].lrow0 == blk[i].lrow0 + n) {
      n += blk[j].nrows;
      ++j;
    }
    runs.push_back({blk[i].lrow0, n});
    i = j;
  }
  return runs;
}

const char *build_plan(const kie_model_desc &m, int n_ctas, size_t smem_cap, Plan &P) {
  const Layout Ly = make_layout(m);
  const int nl = m.n_lanes, d = m.d_model, dh = m.head_dim;
  const int dl = d / nl, hq = m.n_heads / nl, hkv = m.n_kv_heads / nl, fl = m.ffn_dim / nl;
  const int Hkv = m.n_kv_heads, G = m.n_heads / m.n_kv_heads;
  const bool lanes = nl > 1;
  P.n_ctas = n_ctas;
  const char *err = nullptr;
  if ((err = make_shape(dl, d, (m.n_heads + 2 * Hkv) * dh, dl, P.shape[ST_QKV])) ||
      (err = make_cshape(dl, m.n_heads * dh, P.shape[ST_O])) ||
      (err = make_shape(dl, d, m.ffn_dim, dl, P.shape[ST_GU])) ||
      (err = make_cshape(dl, m.ffn_dim, P.shape[ST_D])) ||
      (err = make_shape(d, d, d, 0, P.shape[ST_MIX])) ||
      (err = make_shape(d, d, m.vocab, d, P.shape[ST_LM])))
    return err;
  auto lane0 = [&](int ln) { return Ly.layer0 + int64_t(ln) * Ly.lane_stride; };

  // ---- pass 1: each CTA's rows of each stage, as output blocks
  P.stage_cta.assign(size_t(ST_COUNT) * n_ctas, StageCta{});
  std::vector<std::vector<Block>> oblk(size_t(ST_COUNT) * n_ctas);
  std::vector<std::vector<Piece>> osrc(size_t(ST_COUNT) * n_ctas);
  int longest_run[ST_COUNT] = {};
  for (int c = 0; c < n_ctas; ++c) {
    const int g = c % Hkv, sidx = c / Hkv, ng = (n_ctas - 1 - g) / Hkv + 1;
    const int ln_g = g / hkv;   // lane of KV head g (0 for dense models)
    for (int k = 0; k < ST_COUNT; ++k) {
      if (k == ST_MIX && !lanes) continue;
      StageCta &sc = P.stage_cta[size_t(k) * n_ctas + c];
      const StageShape &sh = P.shape[k];
      std::vector<Piece> pieces;
      int r0 = 0, r1 = 0;
      switch (k) {
        case ST_QKV: {   // q rows of the group's query heads, then its k and v rows
          for (int h = G * g; h < G * (g + 1); ++h)
            pieces.push_back({lane0(ln_g) + Ly.wq + int64_t(h - ln_g * hq) * dh * dl, -1, dh, dl,
                              ln_g * dl, h * dh, 0, 0});
          pieces.push_back({lane0(ln_g) + Ly.wk + int64_t(g - ln_g * hkv) * dh * dl, -1, dh, dl,
                            ln_g * dl, m.n_heads * dh + g * dh, 0, 0});
          pieces.push_back({lane0(ln_g) + Ly.wv + int64_t(g - ln_g * hkv) * dh * dl, -1, dh, dl,
                            ln_g * dl, (m.n_heads + Hkv) * dh + g * dh, 0, 0});
          const int N = (G + 2) * dh;
          r0 = int(int64_t(N) * sidx / ng);
          r1 = int(int64_t(N) * (sidx + 1) / ng);
          break;
        }
        case ST_O: {     // columns of Wo for the group's attention outputs
          pieces.push_back({lane0(ln_g) + Ly.wo + int64_t(G * g * dh - ln_g * hq * dh), -1, G * dh,
                            dl, 0, ln_g * dl, 1, hq * dh});
          const int N = G * dh;
          r0 = int(int64_t(N) * sidx / ng);
          r1 = int(int64_t(N) * (sidx + 1) / ng);
          break;
        }
        case ST_GU:
        case ST_D: {     // this CTA's slice of the hidden units, per lane
          for (int ln = 0; ln < nl; ++ln) {
            if (k == ST_GU)
              pieces.push_back({lane0(ln) + Ly.wg, lane0(ln) + Ly.wu, fl, dl, ln * dl, ln * fl, 0, 0});
            else
              pieces.push_back({lane0(ln) + Ly.wd, -1, fl, dl, 0, ln * dl, 1, fl});
          }
          r0 = int(int64_t(m.ffn_dim) * c / n_ctas);
          r1 = int(int64_t(m.ffn_dim) * (c + 1) / n_ctas);
          break;
        }
        case ST_MIX:
          pieces.push_back({Ly.layer0 + Ly.mix, -1, d, d, 0, 0, 0, 0});
          r0 = int(int64_t(d) * c / n_ctas);
          r1 = int(int64_t(d) * (c + 1) / n_ctas);
          break;
        case ST_LM:
          pieces.push_back({Ly.lm_head, -1, m.vocab, d, 0, 0, 0, 0});
          r0 = int(int64_t(m.vocab) * c / n_ctas);
          r1 = int(int64_t(m.vocab) * (c + 1) / n_ctas);
          break;
      }
      sc.row0 = r0;
      sc.nout = r1 - r0;
      int tile = 0;
      std::vector<Block> &blk = oblk[size_t(k) * n_ctas + c];
      std::vector<Piece> &src = osrc[size_t(k) * n_ctas + c];
      cut_blocks(pieces, r0, r1, false, 0, sh, tile, blk, src);
      if (k == ST_GU) cut_blocks(pieces, r0, r1, true, sc.nout, sh, tile, blk, src);
      sc.nlocal = (k == ST_GU) ? 2 * sc.nout : sc.nout;
      if (sh.cols) {
        sc.ntiles = tile;
        if (sc.nlocal > kMaxLocal) return "too many split-projection rows per CTA";
      } else {
        for (auto &r : input_runs(blk)) longest_run[k] = std::max(longest_run[k], r.second);
        if (k != ST_LM && sc.nlocal > kMaxRowSums) return "too many rows of a row stage per CTA";
      }
      if (k == ST_GU && sc.nout > kMaxLocal) return "hidden slice per CTA too large";
      int64_t bytes = 0;
      for (const Block &B : blk) bytes += int64_t(B.nrows) * sh.K * 2;
      sc.bytes = bytes;
    }
  }
  for (int k = 0; k < ST_COUNT; ++k)
    if (!P.shape[k].cols) set_row_tiling(P.shape[k], longest_run[k]);

  // ---- pass 2: per CTA, its output blocks and row blocks; the streams in
  // consumption order and the repack jobs that fill them
  P.cta_blk_begin.assign(n_ctas + 1, 0);
  int rsum_max = 4;
  int64_t off = 0;
  for (int c = 0; c < n_ctas; ++c) {
    P.cta_blk_begin[c] = int(P.blocks.size());
    int local_blk = 0;
    std::vector<std::vector<Block>> rblk(ST_COUNT);
    for (int k = 0; k < ST_COUNT; ++k) {
      StageCta &sc = P.stage_cta[size_t(k) * n_ctas + c];
      const StageShape &sh = P.shape[k];
      const std::vector<Block> &blk = oblk[size_t(k) * n_ctas + c];
      sc.blk_begin = local_blk;
      sc.nblk = int(blk.size());
      for (const Block &B : blk) P.blocks.push_back(B);
      local_blk += sc.nblk;
      if (sh.cols || (k == ST_MIX && !lanes)) continue;
      // row blocks: each run of one input slice cut into equal parts of <= R rows
      const int kb = 128 * sh.cps, nk = sh.K / kb;
      int tile = 0;
      for (auto &r : input_runs(blk)) {
        const int nb = (r.second + sh.R - 1) / sh.R;
        for (int b = 0; b < nb; ++b) {
          Block R{};
          R.lrow0 = r.first + int(int64_t(r.second) * b / nb);
          R.nrows = r.first + int(int64_t(r.second) * (b + 1) / nb) - R.lrow0;
          R.in_off = blk[0].in_off;
          for (const Block &B : blk)
            if (R.lrow0 >= B.lrow0 && R.lrow0 < B.lrow0 + B.nrows) R.in_off = B.in_off;
          R.tile0 = tile;
          tile += nk;
          rblk[k].push_back(R);
        }
      }
      sc.rb_begin = local_blk;
      sc.nrb = int(rblk[k].size());
      sc.ntiles = tile;
      for (const Block &R : rblk[k]) P.blocks.push_back(R);
      local_blk += sc.nrb;
      if (k != ST_LM) rsum_max = std::max(rsum_max, sc.nlocal);
    }
    if (local_blk > kMaxBlocksPerCta) return "too many row blocks per CTA for this shape";

    P.cta_stream_off.push_back(off);
    auto emit = [&](int k, int64_t layer_off) {
      const StageCta &sc = P.stage_cta[size_t(k) * n_ctas + c];
      const StageShape &sh = P.shape[k];
      const std::vector<Block> &blk = oblk[size_t(k) * n_ctas + c];
      const std::vector<Piece> &src = osrc[size_t(k) * n_ctas + c];
      if (sh.cols) {
        for (int b = 0; b < sc.nblk; ++b) {
          RepackJob j{};
          j.src_elem = src[b].src + layer_off;
          j.dst_byte = off;
          j.nrows = blk[b].nrows;
          j.K = sh.K;
          j.trans = src[b].trans;
          j.src_ld = src[b].ld;
          P.jobs.push_back(j);
          off += int64_t(blk[b].nrows) * sh.K * 2;
        }
        return;
      }
      // a row block's tiles, filled from the output blocks that hold its rows
      for (const Block &R : rblk[k]) {
        for (int b = 0; b < sc.nblk; ++b) {
          const Block &B = blk[b];
          const int lo = std::max(R.lrow0, B.lrow0), hi = std::min(R.lrow0 + R.nrows, B.lrow0 + B.nrows);
          if (lo >= hi) continue;
          RepackJob j{};
          j.src_elem = src[b].src + layer_off + int64_t(lo - B.lrow0) * sh.K;
          j.dst_byte = off;
          j.nrows = hi - lo;
          j.K = sh.K;
          j.trans = 2;
          j.rb = R.nrows;
          j.rb0 = lo - R.lrow0;
          j.kb = 128 * sh.cps;
          P.jobs.push_back(j);
        }
        off += int64_t(R.nrows) * sh.K * 2;
      }
    };
    for (int l = 0; l < m.n_layers; ++l) {
      const int64_t lo = int64_t(l) * Ly.layer_stride;
      emit(ST_QKV, lo);
      if (lanes && l >= 1) emit(ST_MIX, lo - Ly.layer_stride);
      emit(ST_O, lo);
      emit(ST_GU, lo);
      emit(ST_D, lo);
    }
    if (lanes) emit(ST_MIX, int64_t(m.n_layers - 1) * Ly.layer_stride);
    emit(ST_LM, 0);
    off = (off + 255) / 256 * 256;
  }
  P.cta_blk_begin[n_ctas] = int(P.blocks.size());
  P.stream_bytes = off;

  // shared memory: staging / attention scratch, partial sums, ring
  int vb = d;       // staged input of a row stage
  vb = std::max(vb, (G + 2) * dh + kConsumerWarps * G * (dh + 2));   // attention scratch
  vb = std::max(vb, G * std::min((n_ctas + Hkv - 1) / Hkv, kMaxSplit) * (dh + 2));  // group partials
  for (int g = 0; g < Hkv; ++g) {   // merge staging: (m, l) of every split + own output columns
    const int ng = (n_ctas - 1 - g) / Hkv + 1;
    const int nr = (G * dh + ng - 1) / ng;
    vb = std::max(vb, 2 * G * kMaxSplit + std::min(ng, kMaxSplit) * nr);
  }
  for (int k : {int(ST_O), int(ST_D)})                               // column-stage phases
    vb = std::max(vb, P.shape[k].nseg * P.shape[k].K);
  P.vbuf_floats = (vb + 3) / 4 * 4;
  // row stages: the 16 warps' partial sums of two row blocks, then the row
  // sums of the stage (every row stage but the LM head, whose epilogue runs
  // per row block)
  P.rsum_off = kPartialFloats;
  P.part_floats = (kPartialFloats + rsum_max + 3) / 4 * 4;
  const size_t fixed = monokernel_smem_bytes(0, P.vbuf_floats, P.part_floats);
  if (fixed + 3 * (kSlotBytes + 16) > smem_cap) return "shape needs more shared memory than the SM has";
  int slots = int((smem_cap - fixed) / (kSlotBytes + 16));
  slots = std::min(slots, 16);
  // tuning override (never above what shared memory holds)
  if (const char *env = getenv("KIE_RING_SLOTS")) {
    const long v = atol(env);
    if (v >= 2 && v < slots) slots = int(v);
  }
  P.ring_slots = slots;
  P.smem = monokernel_smem_bytes(slots, P.vbuf_floats, P.part_floats);
  P.max_split = std::min((n_ctas + Hkv - 1) / Hkv, kMaxSplit);


  // weights streamed by one decode step: all matrices, norms, one embedding row
  P.weight_bytes_per_step = (Ly.total - int64_t(m.vocab) * d + d) * 2;
  return nullptr;
}

}  // namespace

// ---------------------------------------------------------------- context
struct kie_ctx {
  kie_model_desc m{};
  int device = 0;
  cudaStream_t stream = nullptr;
  Plan plan;
  int pos = 0;
  int pending = -1;
  int poisoned = 0;   // sticky error code
  uint64_t watchdog_ns = 2000000000ull;
  int skip_signal_cta = -1;
  int grid_sync = 0;
  int det_sum = 0;            // KIE_SUM_EXACT: order-independent O / down sums
  int max_launch_steps = 0;   // 0: the counters' own limit (steps_per_launch)
  // L2 look-ahead of the weight producer while its ring is full (KIE_L2PF_TILES,
  // KIE_L2PF_DELAY, KIE_L2PF_PACE): most tiles, cycles before, cycles between
  int l2pf_tiles = 0, l2pf_delay = 2000, l2pf_pace = 600;
  float last_ms = 0.f;
  int last_steps = 0;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  // device buffers
  uint8_t *wstream = nullptr;
  uint16_t *embed = nullptr;
  float *gains = nullptr;  // [2L + 1, d]
  float2 *rope = nullptr;
  uint16_t *kcache = nullptr, *vcache = nullptr;
  float *act = nullptr;    // x, qkv, attn_o, h, u, dsum, attn_part
  uint32_t *sync = nullptr;
  unsigned long long *keys = nullptr;
  int32_t *tokens_in = nullptr, *tokens_out = nullptr;
  StageCta *d_stage_cta = nullptr;
  Block *d_blocks = nullptr;
  int32_t *d_blk_begin = nullptr;
  int64_t *d_stream_off = nullptr;
  unsigned long long *prof = nullptr;  // [n_ctas][kProfSlots] (profiling build)
  unsigned long long *trace = nullptr; // [1 + kTraceCap] (profiling build)
  int trace_cta = 0, trace_step = -1;
  // activation buffer layout (floats): residual bases, the two layer
  // accumulators (both parities, contiguous so one memset clears them), q/k/v,
  // delayed sums, attention partials
  size_t off_xres, off_acc, off_qkv, off_dsum, off_part, act_floats;
  size_t kv_elems = 0;
  std::vector<int32_t> host_tokens;
  // prompt pass on the tensor cores (dense models): the canonical weights as
  // GEMM B operands, their tensor maps (per layer q/k/v, O, gate/up, down,
  // then the LM head), and grow-only scratch for the prompt rows
  int prefill_gemm = 0;           // 1: kie_prefill runs the GEMM prompt pass
  int prefill_gemm_ok = 0;        // the prompt pass is available for this model
  uint16_t *wcanon = nullptr;
  std::vector<CUtensorMap> bmaps;
  int pf_cap = 0, pf_rows_pad = 0;
  float *pf_x = nullptr, *pf_qkv = nullptr, *pf_o = nullptr, *pf_gu = nullptr, *pf_logits = nullptr;
  uint16_t *pf_a = nullptr;       // A parts [P][pf_rows_pad][kmax]
  int32_t *pf_tok = nullptr;      // the prompt, then the greedy token
  uint32_t *pf_status = nullptr;
  float last_prefill_ms = 0.f;
  // sampling at the LM head: the uniforms of a call, the step's logits, each
  // CTA's top-k candidates and its tagged probability sum
  float *uniforms = nullptr, *zbuf = nullptr;
  unsigned long long *cand = nullptr, *psum = nullptr;
  int max_lm_rows = 0;   // LM-head rows of the largest CTA slice
};

static const char *validate(const kie_model_desc *m) {
  if (!m) return "null descriptor";
  if (m->n_layers < 1 || m->d_model < 8 || m->n_heads < 1 || m->n_kv_heads < 1 ||
      m->ffn_dim < 8 || m->vocab < 1 || m->max_seq < 1)
    return "sizes must be positive";
  if (m->head_dim != 64 && m->head_dim != 128) return "head_dim must be 64 or 128";
  if (m->dtype != KIE_F16 && m->dtype != KIE_BF16) return "dtype must be KIE_F16 or KIE_BF16";
  if (m->n_lanes < 1) return "n_lanes must be >= 1";
  if (m->n_heads % m->n_kv_heads) return "n_heads must be a multiple of n_kv_heads";
  if (m->n_heads / m->n_kv_heads > 4) return "at most 4 query heads per KV head";
  const int nl = m->n_lanes;
  if (m->d_model % nl || m->n_heads % nl || m->n_kv_heads % nl || m->ffn_dim % nl)
    return "lane count must divide d_model, heads, kv heads and ffn_dim";
  if (m->n_heads * m->head_dim != m->d_model) return "n_heads * head_dim must equal d_model";
  if ((m->d_model / nl) % 8 || (m->ffn_dim / nl) % 8) return "lane width and lane ffn must be multiples of 8";
  if ((m->d_model / nl) % 128) return "lane width (d_model / n_lanes) must be a multiple of 128";
  if (m->d_model > 4096) return "d_model above 4096 is not supported";
  // rows of d_model (lane mix, LM head) and of the lane width are split over
  // K / 128 lanes of a warp, a power of two
  const int w128 = m->d_model / nl / 128, d128 = m->d_model / 128;
  if ((w128 & (w128 - 1)) || (d128 & (d128 - 1)))
    return "lane width and d_model must be 128 times a power of two";
  if (nl > 1 && m->lane_delay < 2) return "lane_delay must be >= 2";
  if (nl > 64) return "at most 64 lanes";
  if (!(m->rms_eps >= 0.f) || !(m->rope_theta > 0.f)) return "bad rms_eps or rope_theta";
  return nullptr;
}

static int cuda_fail(kie_ctx *c, const char *what, cudaError_t e) {
  set_error(what, e);
  if (c) c->poisoned = KIE_ERR_CUDA;
  return KIE_ERR_CUDA;
}

#define CK(call)                                                    \
  do {                                                              \
    cudaError_t e_ = (call);                                        \
    if (e_ != cudaSuccess) return cuda_fail(ctx, #call, e_);        \
  } while (0)

static void free_ctx(kie_ctx *c) {
  if (!c) return;
  void *ptrs[] = {c->wstream, c->embed, c->gains, c->rope, c->kcache, c->vcache, c->act,
                  c->sync, c->keys, c->tokens_in, c->tokens_out, c->d_stage_cta, c->d_blocks,
                  c->d_blk_begin, c->d_stream_off, c->prof, c->trace, c->wcanon, c->pf_x,
                  c->pf_qkv, c->pf_o, c->pf_gu, c->pf_logits, c->pf_a, c->pf_tok, c->pf_status,
                  c->uniforms, c->zbuf, c->cand, c->psum};
  for (void *p : ptrs)
    if (p) cudaFree(p);
  if (c->ev0) cudaEventDestroy(c->ev0);
  if (c->ev1) cudaEventDestroy(c->ev1);
  delete c;
}

static int alloc(kie_ctx *ctx, void **p, size_t bytes, const char *what) {
  cudaError_t e = cudaMalloc(p, bytes ? bytes : 16);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    set_error(what, e);
    return KIE_ERR_OOM;
  }
  if (e != cudaSuccess) return cuda_fail(ctx, what, e);
  return KIE_OK;
}

// ---------------------------------------------------------------- prompt pass (tensor cores)
// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time
// dependency on the driver library).
static PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// Tensor map of a row-major [rows, K] matrix of 16-bit words with row pitch
// ld elements, read as 64-column x 128-row boxes with 128-byte swizzle (the
// GEMM's operand tiles); columns >= K and rows >= rows read as zero.
static bool make_tmap(CUtensorMap *map, const void *base, int dtype, int64_t K, int64_t rows, int64_t ld) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encode_fn();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15) || ((ld * 2) & 15)) return false;
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {cuuint32_t(gemm_tile_k()), cuuint32_t(gemm_tile_m())};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dtype == KIE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

extern "C" int kie_weights_bytes(const kie_model_desc *desc, int64_t *out) {
  if (!out) return KIE_ERR_INVALID;
  if (const char *why = validate(desc)) {
    g_last_error = why;
    return KIE_ERR_INVALID;
  }
  *out = make_layout(*desc).total * 2;
  return KIE_OK;
}

static InstShape inst_shape(const kie_model_desc &m, const Plan &P);

extern "C" int kie_create(const kie_model_desc *desc, const void *weights, void *stream,
                          kie_ctx **out) {
  if (!out) return KIE_ERR_INVALID;
  *out = nullptr;
  if (const char *why = validate(desc)) {
    g_last_error = why;
    return KIE_ERR_INVALID;
  }
  if (!weights || (reinterpret_cast<uintptr_t>(weights) & 15)) {
    g_last_error = "weights must be a 16-byte aligned device pointer";
    return KIE_ERR_INVALID;
  }
  kie_ctx *ctx = new kie_ctx();
  ctx->m = *desc;
  ctx->stream = static_cast<cudaStream_t>(stream);
  const kie_model_desc &m = ctx->m;
  int rc;
  auto fail = [&](int code) {
    free_ctx(ctx);
    return code;
  };
  if (const char *env = getenv("KIE_WATCHDOG_MS")) {
    long v = atol(env);
    if (v > 0) ctx->watchdog_ns = uint64_t(v) * 1000000ull;
  }
  // tuning overrides of the L2 look-ahead (clamped to sane ranges)
  if (const char *env = getenv("KIE_L2PF_TILES")) ctx->l2pf_tiles = std::max(0, std::min(64, atoi(env)));
  if (const char *env = getenv("KIE_L2PF_DELAY")) ctx->l2pf_delay = std::max(0, std::min(1 << 24, atoi(env)));
  if (const char *env = getenv("KIE_L2PF_PACE")) ctx->l2pf_pace = std::max(0, std::min(1 << 24, atoi(env)));
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e != cudaSuccess) return fail(cuda_fail(nullptr, "cudaGetDevice", e));
  cudaPointerAttributes pa{};
  e = cudaPointerGetAttributes(&pa, weights);
  if (e != cudaSuccess || (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)) {
    cudaGetLastError();
    g_last_error = "weights is not a device pointer";
    return fail(KIE_ERR_INVALID);
  }
  int n_sm = 0, smem_optin = 0, coop = 0;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, ctx->device);
  cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, ctx->device);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, ctx->device);
  if (!coop) {
    g_last_error = "device lacks cooperative launch";
    return fail(KIE_ERR_NOT_RESIDENT);
  }
  if (n_sm < m.n_kv_heads) {
    g_last_error = "fewer SMs than KV heads";
    return fail(KIE_ERR_NOT_RESIDENT);
  }
  if (const char *why = build_plan(m, n_sm, size_t(smem_optin), ctx->plan)) {
    g_last_error = why;
    return fail(KIE_ERR_INVALID);
  }
  Plan &P = ctx->plan;
  for (int variant = 0; variant < 5; ++variant) {   // every kernel instance this model can launch
    const void *fn = monokernel_fn(m.dtype, variant, inst_shape(m, P));
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(P.smem));
    if (e != cudaSuccess) return fail(cuda_fail(nullptr, "cudaFuncSetAttribute", e));
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, monokernel_threads(), P.smem);
    if (e != cudaSuccess) return fail(cuda_fail(nullptr, "occupancy query", e));
    if (per_sm < 1) {
      g_last_error = "persistent CTA does not fit on an SM";
      return fail(KIE_ERR_NOT_RESIDENT);
    }
  }

  const Layout Ly = make_layout(m);
  const int d = m.d_model, L = m.n_layers, dh = m.head_dim;
  // ---- allocations
  if ((rc = alloc(ctx, (void **)&ctx->wstream, P.stream_bytes, "weight stream"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->embed, size_t(m.vocab) * d * 2, "embedding"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->gains, size_t(2 * L + 1) * d * 4, "gains"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->rope, size_t(m.max_seq) * (dh / 2) * 8, "rope"))) return fail(rc);
  ctx->kv_elems = size_t(L) * m.n_kv_heads * m.max_seq * dh;
  if ((rc = alloc(ctx, (void **)&ctx->kcache, ctx->kv_elems * 2, "K cache"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->vcache, ctx->kv_elems * 2, "V cache"))) return fail(rc);
  size_t o = 0;
  auto take = [&](size_t n) { size_t r = o; o += (n + 63) / 64 * 64; return r; };
  ctx->off_xres = take(size_t(2) * d);
  ctx->off_acc = take(size_t(8) * d);   // acc_o[2][d] then acc_d[2][d], each with room for lo sums
  // tagged words (8 bytes: two floats' room each)
  ctx->off_qkv = take(size_t(2) * (m.n_heads + 2 * m.n_kv_heads) * dh);
  ctx->off_dsum = take(size_t(std::max(1, m.lane_delay)) * d);
  ctx->off_part = take(size_t(2) * m.n_heads * P.max_split * (dh + 2));
  ctx->act_floats = o;
  if ((rc = alloc(ctx, (void **)&ctx->act, o * 4, "activations"))) return fail(rc);
  const size_t sync_words = size_t(SY_COUNT) * kSyncStride;
  if ((rc = alloc(ctx, (void **)&ctx->sync, sync_words * 4, "sync"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->keys, size_t(m.max_seq) * 8, "keys"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->tokens_in, size_t(m.max_seq) * 4, "tokens"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->tokens_out, size_t(m.max_seq) * 4, "tokens"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->uniforms, size_t(m.max_seq) * 4, "sampling"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->zbuf, size_t(m.vocab) * 4, "sampling"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->cand, size_t(P.n_ctas) * kMaxTopK * 8, "sampling"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->psum, size_t(P.n_ctas) * 8, "sampling"))) return fail(rc);
  for (int c = 0; c < P.n_ctas; ++c)
    ctx->max_lm_rows = std::max(ctx->max_lm_rows, P.stage_cta[size_t(ST_LM) * P.n_ctas + c].nout);
  if ((rc = alloc(ctx, (void **)&ctx->d_stage_cta, P.stage_cta.size() * sizeof(StageCta), "plan"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->d_blocks, std::max<size_t>(1, P.blocks.size()) * sizeof(Block), "plan"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->d_blk_begin, P.cta_blk_begin.size() * 4, "plan"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->d_stream_off, P.cta_stream_off.size() * 8, "plan"))) return fail(rc);
  if ((rc = alloc(ctx, (void **)&ctx->prof, size_t(P.n_ctas) * kProfSlots * 8, "profile"))) return fail(rc);
  if (monokernel_profiled() &&
      (rc = alloc(ctx, (void **)&ctx->trace, size_t(kTraceCap + 1) * 8, "trace"))) return fail(rc);
  RepackJob *d_jobs = nullptr;
  if ((rc = alloc(ctx, (void **)&d_jobs, P.jobs.size() * sizeof(RepackJob), "repack jobs"))) return fail(rc);

  cudaStream_t st = ctx->stream;
  auto ck = [&](cudaError_t er, const char *what) {
    if (er != cudaSuccess) { cuda_fail(nullptr, what, er); return false; }
    return true;
  };
  bool ok = true;
  ok = ok && ck(cudaMemcpyAsync(ctx->d_stage_cta, P.stage_cta.data(), P.stage_cta.size() * sizeof(StageCta), cudaMemcpyHostToDevice, st), "plan copy");
  if (!P.blocks.empty())
    ok = ok && ck(cudaMemcpyAsync(ctx->d_blocks, P.blocks.data(), P.blocks.size() * sizeof(Block), cudaMemcpyHostToDevice, st), "plan copy");
  ok = ok && ck(cudaMemcpyAsync(ctx->d_blk_begin, P.cta_blk_begin.data(), P.cta_blk_begin.size() * 4, cudaMemcpyHostToDevice, st), "plan copy");
  ok = ok && ck(cudaMemcpyAsync(ctx->d_stream_off, P.cta_stream_off.data(), P.cta_stream_off.size() * 8, cudaMemcpyHostToDevice, st), "plan copy");
  ok = ok && ck(cudaMemcpyAsync(d_jobs, P.jobs.data(), P.jobs.size() * sizeof(RepackJob), cudaMemcpyHostToDevice, st), "plan copy");
  const uint16_t *w = static_cast<const uint16_t *>(weights);
  ok = ok && ck(launch_repack(w, ctx->wstream, d_jobs, int(P.jobs.size()), st), "repack");
  ok = ok && ck(cudaMemcpyAsync(ctx->embed, w + Ly.embed, size_t(m.vocab) * d * 2, cudaMemcpyDeviceToDevice, st), "embedding copy");
  // norm gains: widen to fp32 on the host (exact) from a host copy of the gain words
  std::vector<uint16_t> gbits(size_t(2 * L + 1) * d);
  const int nl = m.n_lanes, dl = d / nl;
  for (int l = 0; l < L && ok; ++l)
    for (int ln = 0; ln < nl && ok; ++ln) {
      const int64_t lane0 = Ly.layer0 + int64_t(l) * Ly.layer_stride + int64_t(ln) * Ly.lane_stride;
      ok = ck(cudaMemcpyAsync(&gbits[size_t(l) * d + size_t(ln) * dl], w + lane0 + Ly.attn_norm, size_t(dl) * 2, cudaMemcpyDeviceToHost, st), "gain copy") &&
           ck(cudaMemcpyAsync(&gbits[size_t(L + l) * d + size_t(ln) * dl], w + lane0 + Ly.ffn_norm, size_t(dl) * 2, cudaMemcpyDeviceToHost, st), "gain copy");
    }
  ok = ok && ck(cudaMemcpyAsync(&gbits[size_t(2 * L) * d], w + Ly.final_norm, size_t(d) * 2, cudaMemcpyDeviceToHost, st), "gain copy");
  ok = ok && ck(cudaStreamSynchronize(st), "create sync");
  if (!ok) { cudaFree(d_jobs); return fail(KIE_ERR_CUDA); }
  std::vector<float> gains(gbits.size());
  for (size_t i = 0; i < gbits.size(); ++i) {
    const uint32_t b = gbits[i];
    if (m.dtype == KIE_BF16) {
      uint32_t u = b << 16;
      memcpy(&gains[i], &u, 4);
    } else {  // binary16 -> binary32, from the format definition
      const uint32_t s = (b >> 15) & 1, ex = (b >> 10) & 31, fr = b & 1023;
      float v;
      if (ex == 0) v = ldexpf(float(fr), -24);
      else if (ex == 31) v = fr ? NAN : INFINITY;
      else v = ldexpf(float(fr | 1024), int(ex) - 25);
      gains[i] = s ? -v : v;
    }
  }
  // RoPE table: angle p * theta^(-2i/dh) and its cos/sin in double, stored fp32
  std::vector<float2> rope(size_t(m.max_seq) * (dh / 2));
  for (int p = 0; p < m.max_seq; ++p)
    for (int i = 0; i < dh / 2; ++i) {
      const double ang = double(p) * pow(double(m.rope_theta), -2.0 * i / dh);
      rope[size_t(p) * (dh / 2) + i] = make_float2(float(cos(ang)), float(sin(ang)));
    }
  ok = ck(cudaMemcpyAsync(ctx->gains, gains.data(), gains.size() * 4, cudaMemcpyHostToDevice, st), "gain upload") &&
       ck(cudaMemcpyAsync(ctx->rope, rope.data(), rope.size() * 8, cudaMemcpyHostToDevice, st), "rope upload") &&
       ck(cudaMemsetAsync(ctx->kcache, 0xff, ctx->kv_elems * 2, st), "cache poison") &&
       ck(cudaMemsetAsync(ctx->vcache, 0xff, ctx->kv_elems * 2, st), "cache poison") &&
       ck(cudaMemsetAsync(ctx->act, 0, ctx->act_floats * 4, st), "act clear") &&
       ck(cudaEventCreate(&ctx->ev0), "event") && ck(cudaEventCreate(&ctx->ev1), "event") &&
       ck(cudaStreamSynchronize(st), "create sync");
  cudaFree(d_jobs);
  if (!ok) return fail(KIE_ERR_CUDA);
  // the tensor-core prompt pass (dense models): a canonical copy of the
  // weights for its GEMM operands; without room for it, prompts run through
  // the persistent kernel one position per step
  if (m.n_lanes == 1 && cudaMalloc((void **)&ctx->wcanon, size_t(Ly.total) * 2) == cudaSuccess) {
    bool mk = ck(cudaMemcpyAsync(ctx->wcanon, w, size_t(Ly.total) * 2, cudaMemcpyDeviceToDevice, st),
                 "weights copy") && ck(cudaStreamSynchronize(st), "create sync");
    if (!mk) return fail(KIE_ERR_CUDA);
    const int64_t nq = int64_t(m.n_heads + 2 * m.n_kv_heads) * dh, hd = int64_t(m.n_heads) * dh;
    ctx->bmaps.resize(size_t(4) * L + 1);
    for (int l = 0; l < L && mk; ++l) {
      const uint16_t *lw = ctx->wcanon + Ly.layer0 + int64_t(l) * Ly.layer_stride;
      mk = make_tmap(&ctx->bmaps[4 * l + 0], lw + Ly.wq, m.dtype, d, nq, d) &&
           make_tmap(&ctx->bmaps[4 * l + 1], lw + Ly.wo, m.dtype, hd, d, hd) &&
           make_tmap(&ctx->bmaps[4 * l + 2], lw + Ly.wg, m.dtype, d, 2 * int64_t(m.ffn_dim), d) &&
           make_tmap(&ctx->bmaps[4 * l + 3], lw + Ly.wd, m.dtype, m.ffn_dim, d, m.ffn_dim);
    }
    mk = mk && make_tmap(&ctx->bmaps[4 * L], ctx->wcanon + Ly.lm_head, m.dtype, d, m.vocab, d);
    // default: the tensor-core pass for fp16 models; bf16 models keep the
    // decode path's own per-position prompt, whose cache matches the oracle's
    // more closely (bf16 rounding turns fp32-level differences of the pass's
    // tensor-core accumulation into one-ulp flips of cached K/V)
    ctx->prefill_gemm_ok = mk ? 1 : 0;
    ctx->prefill_gemm = mk && m.dtype == KIE_F16 ? 1 : 0;
    if (!mk) {
      cudaFree(ctx->wcanon);
      ctx->wcanon = nullptr;
    }
  }
  cudaGetLastError();
  *out = ctx;
  return KIE_OK;
}

// Run the persistent kernel for n steps from position pos0.
// Turns the kernel's status word into a kie_status and poisons the context:
// the launch left mid-step, so the KV cache and position are not consistent.
// Low byte: 1..3 a bounded wait ran out (which counter or barrier in the next
// byte), 4 a NaN logit or an out-of-range token id (step in bits 8..23).
static int device_error(kie_ctx *ctx, uint32_t status) {
  char buf[160];
  const uint32_t kind = status & 0xffu;
  const int rc = kind == 4u ? KIE_ERR_NONFINITE : KIE_ERR_DEVICE_TIMEOUT;
  if (kind == 4u)
    snprintf(buf, sizeof buf, "non-finite logits or token id out of range at step %u (code 0x%x)",
             status >> 8, status);
  else
    snprintf(buf, sizeof buf, "device watchdog: a bounded wait ran out (code 0x%x)", status);
  g_last_error = buf;
  ctx->poisoned = rc;
  return rc;
}

// The epoch counters are 32-bit, and every CTA adds to them at most 4 L + 2
// times per step: the q/k/v, attention, O and down signals of each layer, and
// the lane-mix flush and token of each step.  One launch therefore runs at
// most this many steps, so that no counter passes 2^31; a longer call runs as
// several launches back to back.
static int steps_per_launch(const kie_ctx *ctx) {
  const int64_t per_step = (4 * int64_t(ctx->m.n_layers) + 2) * ctx->plan.n_ctas;
  int64_t n = ((int64_t(1) << 31) - 1) / per_step;
  if (ctx->max_launch_steps > 0 && ctx->max_launch_steps < n) n = ctx->max_launch_steps;
  return int(std::max<int64_t>(n, 1));
}

// The model's attention shape and its plan's GEMV widths, as a kernel
// instance may fix them.
static InstShape inst_shape(const kie_model_desc &m, const Plan &P) {
  InstShape k{};
  k.G = m.n_heads / m.n_kv_heads;
  k.dh = m.head_dim;
  k.cq = P.shape[ST_QKV].cps;
  k.cr = P.shape[ST_GU].cps == P.shape[ST_LM].cps ? P.shape[ST_GU].cps : 0;
  k.cc = P.shape[ST_O].cps == P.shape[ST_D].cps ? P.shape[ST_O].cps : 0;
  k.cm = m.n_lanes > 1 ? P.shape[ST_MIX].cps : 0;
  return k;
}

// The kernel instance for these arguments: the general one when an
// ablation switch or the L2 look-ahead is on, or a lane model samples; the
// lanes one for other lane-model calls; else the dense one; with the
// sampler compiled in when a temperature is set.
static int kernel_variant(const KernelArgs &a) {
  const bool ablations = a.grid_sync || a.det_sum || a.l2pf_tiles > 0;
  const bool lanes = a.n_lanes > 1, sample = a.sample_t > 0.f;
  if (ablations || (lanes && sample)) return 1 | (sample ? 2 : 0);
  if (lanes) return 4;
  return sample ? 2 : 0;
}

// Runs the n steps described by `a` (forced tokens, output tokens, argmax
// keys and logits of the whole call) as one or more launches.  Each launch
// takes the next run of steps and starts from the previous launch's last
// token.  The counters, both layer accumulators and the launch's keys are
// cleared before each launch.  The output tokens end in host_out.  The
// context's device time spans from the first launch's start to the last
// one's end.
static int launch_steps(kie_ctx *ctx, const KernelArgs &a, size_t sync_bytes, int n,
                        int32_t *host_out) {
  cudaStream_t st = ctx->stream;
  const int cap = steps_per_launch(ctx);
  int32_t tok = a.first_token;
  uint32_t status = 0;
  for (int s0 = 0; s0 < n; s0 += cap) {
    const int c = std::min(cap, n - s0);
    KernelArgs b = a;
    b.pos0 = a.pos0 + s0;
    b.n_steps = c;
    b.first_token = tok;
    b.forced = a.forced ? a.forced + s0 : nullptr;
    b.out_tokens = a.out_tokens + s0;
    b.keys = a.keys + s0;
    b.uniforms = a.uniforms ? a.uniforms + s0 : nullptr;
    if (a.logits_every_step) {   // every step's logits, each launch at its own offset
      b.logits_out = a.logits_out ? a.logits_out + size_t(s0) * ctx->m.vocab : nullptr;
      b.logits_step0 = 0;
    } else {                     // a prompt: the logits of its last position only
      b.logits_out = s0 + c == n ? a.logits_out : nullptr;
      b.logits_step0 = c - 1;
    }
    b.skip_signal_cta = s0 == 0 ? a.skip_signal_cta : -1;
    if (a.trace && a.trace_step >= s0 && a.trace_step < s0 + c) b.trace_step = a.trace_step - s0;
    else b.trace = nullptr;
    CK(cudaMemsetAsync(a.sync, 0, sync_bytes, st));
    CK(cudaMemsetAsync(a.acc_o, 0, size_t(8) * ctx->m.d_model * 4, st));   // both accumulators, both parities
    CK(cudaMemsetAsync(b.keys, 0, size_t(c) * 8, st));
    // tagged q/k/v and attention partials: tags restart with every launch
    const kie_model_desc &m = ctx->m;
    CK(cudaMemsetAsync(a.qkv, 0, size_t(m.n_heads + 2 * m.n_kv_heads) * m.head_dim * 8, st));
    CK(cudaMemsetAsync(a.attn_part, 0, size_t(m.n_heads) * ctx->plan.max_split * (m.head_dim + 2) * 8, st));
    if (a.sample_t > 0.f) CK(cudaMemsetAsync(a.psum, 0, size_t(ctx->plan.n_ctas) * 8, st));
    if (s0 == 0) CK(cudaEventRecord(ctx->ev0, st));
    void *args[] = {&b};
    CK(cudaLaunchCooperativeKernel(monokernel_fn(ctx->m.dtype, kernel_variant(a), inst_shape(m, ctx->plan)),
                                   dim3(ctx->plan.n_ctas),
                                   dim3(monokernel_threads()), args, ctx->plan.smem, st));
    if (s0 + c < n) {   // the next launch needs this one's last token
      CK(cudaMemcpyAsync(&status, a.sync + SY_STATUS * kSyncStride, 4, cudaMemcpyDeviceToHost, st));
      CK(cudaMemcpyAsync(&tok, b.out_tokens + c - 1, 4, cudaMemcpyDeviceToHost, st));
      CK(cudaStreamSynchronize(st));
      if (status != 0) return device_error(ctx, status);
    }
  }
  CK(cudaEventRecord(ctx->ev1, st));
  CK(cudaMemcpyAsync(&status, a.sync + SY_STATUS * kSyncStride, 4, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(host_out, a.out_tokens, size_t(n) * 4, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  CK(cudaEventElapsedTime(&ctx->last_ms, ctx->ev0, ctx->ev1));
  ctx->last_steps = n;
  if (status != 0) return device_error(ctx, status);
  return KIE_OK;
}

// Kernel arguments of one call: the model, the plan, the weights, the KV
// cache and the context's settings.  The caller points the per-launch scratch
// (activations, counters, keys, token buffers) somewhere and sets the run
// fields it needs beyond pos0 / n / first token / logits.  The pending test
// hook (skip_signal_cta) is consumed here, so it applies to exactly one call.
static KernelArgs fill_args(kie_ctx *ctx, int pos0, int n, int first_token,
                            bool logits_every_step, float *logits_out) {
  const kie_model_desc &m = ctx->m;
  const Plan &P = ctx->plan;
  KernelArgs a{};
  a.n_layers = m.n_layers; a.d_model = m.d_model; a.n_heads = m.n_heads;
  a.n_kv_heads = m.n_kv_heads; a.head_dim = m.head_dim; a.ffn_dim = m.ffn_dim; a.vocab = m.vocab;
  a.n_lanes = m.n_lanes; a.lane_delay = m.n_lanes > 1 ? m.lane_delay : 1;
  a.lane_width = m.d_model / m.n_lanes; a.lane_heads = m.n_heads / m.n_lanes;
  a.lane_kv_heads = m.n_kv_heads / m.n_lanes; a.lane_ffn = m.ffn_dim / m.n_lanes;
  a.rms_eps = m.rms_eps;
  a.attn_scale = float(1.0 / sqrt(double(m.head_dim)));
  a.max_seq = m.max_seq;
  a.n_ctas = P.n_ctas; a.ring_slots = P.ring_slots;
  a.vbuf_floats = P.vbuf_floats; a.part_floats = P.part_floats;
  a.rsum_off = P.rsum_off;
  for (int k = 0; k < ST_COUNT; ++k) a.shape[k] = P.shape[k];
  a.stage_cta = ctx->d_stage_cta; a.blocks = ctx->d_blocks;
  a.cta_blk_begin = ctx->d_blk_begin; a.cta_stream_off = ctx->d_stream_off;
  a.wstream = ctx->wstream; a.embed = ctx->embed;
  a.gain_attn = ctx->gains; a.gain_ffn = ctx->gains + size_t(m.n_layers) * m.d_model;
  a.gain_final = ctx->gains + size_t(2 * m.n_layers) * m.d_model;
  a.rope_cs = ctx->rope; a.kcache = ctx->kcache; a.vcache = ctx->vcache;
  a.max_split = P.max_split;
  a.pos0 = pos0; a.n_steps = n; a.first_token = first_token;
  a.logits_every_step = logits_every_step ? 1 : 0;
  a.logits_out = logits_out;
  a.watchdog_ns = ctx->watchdog_ns;
  a.skip_signal_cta = ctx->skip_signal_cta;
  ctx->skip_signal_cta = -1;
  a.grid_sync = ctx->grid_sync;
  a.det_sum = ctx->det_sum;
  a.l2pf_tiles = ctx->l2pf_tiles; a.l2pf_delay = ctx->l2pf_delay; a.l2pf_pace = ctx->l2pf_pace;
  a.sample_t = 0.f; a.sample_k = 0; a.sample_p = 1.f;   // greedy unless a sampling call says otherwise
  a.zbuf = ctx->zbuf; a.cand = ctx->cand; a.psum = ctx->psum;
  return a;
}

// Points the kernel's per-launch activation scratch at `act` (laid out as the
// context's activation buffer).
static void set_act(const kie_ctx *ctx, KernelArgs &a, float *act) {
  a.xres = act + ctx->off_xres;
  // fp32 sums take [2][d] floats per accumulator, deterministic sums [2][d] hi + [2][d] lo
  a.acc_o = act + ctx->off_acc; a.acc_d = a.acc_o + (ctx->det_sum ? 4 : 2) * size_t(ctx->m.d_model);
  a.qkv = reinterpret_cast<unsigned long long *>(act + ctx->off_qkv);
  a.dsum = act + ctx->off_dsum;
  a.attn_part = reinterpret_cast<unsigned long long *>(act + ctx->off_part);
}

static int run(kie_ctx *ctx, int pos0, int n, const int32_t *forced_host, int first_token,
               bool logits_every_step, float *logits_out, int32_t *out_host,
               const kie_sampling *smp = nullptr, const float *uniforms_host = nullptr) {
  cudaStream_t st = ctx->stream;
  KernelArgs a = fill_args(ctx, pos0, n, first_token, logits_every_step, logits_out);
  if (smp && smp->temperature > 0.f) {
    a.sample_t = smp->temperature;
    a.sample_k = smp->top_k;
    a.sample_p = smp->top_p;
    a.uniforms = ctx->uniforms;
    CK(cudaMemcpyAsync(ctx->uniforms, uniforms_host, size_t(n) * 4, cudaMemcpyHostToDevice, st));
  }
  set_act(ctx, a, ctx->act);
  a.sync = ctx->sync; a.keys = ctx->keys;
  a.forced = forced_host ? ctx->tokens_in : nullptr;
  a.out_tokens = ctx->tokens_out;
  a.prof = ctx->prof;
  if (ctx->trace && ctx->trace_step >= 0 && ctx->trace_step < n) {
    a.trace = ctx->trace;
    a.trace_cap = kTraceCap;
    a.trace_cta = ctx->trace_cta;
    a.trace_step = ctx->trace_step;
    CK(cudaMemsetAsync(ctx->trace, 0, 8, st));
  }

  const size_t sync_bytes = size_t(SY_COUNT) * kSyncStride * 4;
  if (forced_host)
    CK(cudaMemcpyAsync(ctx->tokens_in, forced_host, size_t(n) * 4, cudaMemcpyHostToDevice, st));
  ctx->host_tokens.resize(n);
  if (int rc = launch_steps(ctx, a, sync_bytes, n, ctx->host_tokens.data())) return rc;
  if (out_host) memcpy(out_host, ctx->host_tokens.data(), size_t(n) * 4);
  return KIE_OK;
}

// Grows the prompt pass's scratch to hold n prompt rows.
static int prefill_scratch(kie_ctx *ctx, int n) {
  if (n <= ctx->pf_cap) return KIE_OK;
  const kie_model_desc &m = ctx->m;
  const int d = m.d_model, dh = m.head_dim, F = m.ffn_dim;
  const int P = m.dtype == KIE_F16 ? 2 : 3;
  const size_t nq = size_t(m.n_heads + 2 * m.n_kv_heads) * dh, hd = size_t(m.n_heads) * dh;
  const size_t kmax = std::max<size_t>({size_t(d), hd, size_t(F)});
  const int rows_pad = (n + gemm_tile_m() - 1) / gemm_tile_m() * gemm_tile_m();
  void *bufs[] = {ctx->pf_x, ctx->pf_qkv, ctx->pf_o, ctx->pf_gu, ctx->pf_logits, ctx->pf_a, ctx->pf_tok,
                  ctx->pf_status};
  for (void *b : bufs)
    if (b) cudaFree(b);
  ctx->pf_x = ctx->pf_qkv = ctx->pf_o = ctx->pf_gu = ctx->pf_logits = nullptr;
  ctx->pf_a = nullptr;
  ctx->pf_tok = nullptr;
  ctx->pf_status = nullptr;
  ctx->pf_cap = 0;
  int rc;
  if ((rc = alloc(ctx, (void **)&ctx->pf_x, size_t(n) * d * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_qkv, size_t(n) * nq * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_o, size_t(n) * hd * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_gu, size_t(n) * 2 * F * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_logits, size_t(m.vocab) * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_a, size_t(P) * rows_pad * kmax * 2, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_tok, size_t(n + 1) * 4, "prompt scratch")) ||
      (rc = alloc(ctx, (void **)&ctx->pf_status, 4, "prompt scratch")))
    return rc;
  ctx->pf_cap = n;
  ctx->pf_rows_pad = rows_pad;
  return KIE_OK;
}

// The prompt pass on the tensor cores: every layer for all n prompt rows at
// once (RMSNorm -> q/k/v GEMM -> RoPE + K/V cache -> causal attention -> O
// GEMM into the residual -> RMSNorm -> gate/up GEMM -> SwiGLU -> down GEMM
// into the residual), then the final norm and LM head of the last row and
// its greedy token.  logits_out (device [V] or null) receives that row's
// logits.
static int prefill_gemm_run(kie_ctx *ctx, const int32_t *tokens, int n, float *logits_out, int32_t *next) {
  const kie_model_desc &m = ctx->m;
  const int d = m.d_model, dh = m.head_dim, Hq = m.n_heads, Hkv = m.n_kv_heads, F = m.ffn_dim, L = m.n_layers;
  const int V = m.vocab, P = m.dtype == KIE_F16 ? 2 : 3;
  const int nq = (Hq + 2 * Hkv) * dh, hd = Hq * dh;
  cudaStream_t st = ctx->stream;
  if (int rc = prefill_scratch(ctx, n)) return rc;
  const int64_t kmax = std::max({int64_t(d), int64_t(hd), int64_t(F)});
  const int64_t pstride = int64_t(ctx->pf_rows_pad) * kmax;   // elements between A parts
  CUtensorMap map_ad, map_af;   // the A parts read with K = d and with K = F
  if (!make_tmap(&map_ad, ctx->pf_a, m.dtype, d, int64_t(P) * ctx->pf_rows_pad, kmax) ||
      !make_tmap(&map_af, ctx->pf_a, m.dtype, F, int64_t(P) * ctx->pf_rows_pad, kmax)) {
    g_last_error = "tensor map of the prompt pass could not be encoded";
    ctx->poisoned = KIE_ERR_CUDA;
    return KIE_ERR_CUDA;
  }
  GemmArgs g{};
  g.parts = P;
  g.stages = gemm_stages(P);
  g.a_part_rows = ctx->pf_rows_pad;
  g.dtype = m.dtype;
  g.status = ctx->pf_status;
  g.watchdog_ns = ctx->watchdog_ns;
  auto gemm = [&](const CUtensorMap &ma, const CUtensorMap &mb, int M, int N, int K, float *C, int64_t ldc,
                  int acc) {
    GemmArgs a = g;
    a.M = M; a.N = N; a.K = K; a.C = C; a.ldc = ldc; a.accumulate = acc;
    return launch_gemm(ma, mb, a, st);
  };
  const float *gain_attn = ctx->gains, *gain_ffn = ctx->gains + size_t(L) * d;
  const float *gain_final = ctx->gains + size_t(2 * L) * d;
  const float scale = float(1.0 / sqrt(double(dh)));
  CK(cudaEventRecord(ctx->ev0, st));
  CK(cudaMemcpyAsync(ctx->pf_tok, tokens, size_t(n) * 4, cudaMemcpyHostToDevice, st));
  CK(cudaMemsetAsync(ctx->pf_status, 0, 4, st));
  CK(launch_embed_rows(ctx->embed, ctx->pf_tok, n, d, m.dtype, ctx->pf_x, st));
  for (int l = 0; l < L; ++l) {
    CK(launch_norm_split(ctx->pf_x, gain_attn + size_t(l) * d, n, d, m.rms_eps, P, m.dtype, ctx->pf_a, pstride,
                         kmax, st));
    CK(gemm(map_ad, ctx->bmaps[4 * l + 0], n, nq, d, ctx->pf_qkv, nq, 0));
    CK(launch_rope_kv(ctx->pf_qkv, n, 0, Hq, Hkv, dh, ctx->rope, ctx->kcache, ctx->vcache, l, m.max_seq, m.dtype,
                      scale, st));
    CK(launch_prefill_attention(ctx->pf_qkv, n, 0, Hq, Hkv, dh, ctx->kcache, ctx->vcache, l, m.max_seq, m.dtype,
                                ctx->pf_o, st));
    CK(launch_split(ctx->pf_o, n, hd, hd, P, m.dtype, ctx->pf_a, pstride, kmax, st));
    CK(gemm(map_ad, ctx->bmaps[4 * l + 1], n, d, hd, ctx->pf_x, d, 1));
    CK(launch_norm_split(ctx->pf_x, gain_ffn + size_t(l) * d, n, d, m.rms_eps, P, m.dtype, ctx->pf_a, pstride,
                         kmax, st));
    CK(gemm(map_ad, ctx->bmaps[4 * l + 2], n, 2 * F, d, ctx->pf_gu, 2 * int64_t(F), 0));
    CK(launch_swiglu_split(ctx->pf_gu, n, F, P, m.dtype, ctx->pf_a, pstride, kmax, st));
    CK(gemm(map_af, ctx->bmaps[4 * l + 3], n, d, F, ctx->pf_x, d, 1));
  }
  CK(launch_norm_split(ctx->pf_x + size_t(n - 1) * d, gain_final, 1, d, m.rms_eps, P, m.dtype, ctx->pf_a, pstride,
                       kmax, st));
  CK(gemm(map_ad, ctx->bmaps[4 * L], 1, V, d, ctx->pf_logits, V, 0));
  CK(launch_argmax_row(ctx->pf_logits, V, ctx->pf_tok + n, st));
  if (logits_out)
    CK(cudaMemcpyAsync(logits_out, ctx->pf_logits, size_t(V) * 4, cudaMemcpyDeviceToDevice, st));
  CK(cudaEventRecord(ctx->ev1, st));
  int32_t tok = -1;
  uint32_t status = 0;
  CK(cudaMemcpyAsync(&tok, ctx->pf_tok + n, 4, cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(&status, ctx->pf_status, 4, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  CK(cudaEventElapsedTime(&ctx->last_prefill_ms, ctx->ev0, ctx->ev1));
  if (status != 0) {
    char buf[160];
    snprintf(buf, sizeof buf, "prompt pass: a bounded wait ran out (code 0x%x)", status);
    g_last_error = buf;
    ctx->poisoned = KIE_ERR_DEVICE_TIMEOUT;
    return KIE_ERR_DEVICE_TIMEOUT;
  }
  if (tok < 0 || tok >= V) {
    g_last_error = "non-finite logits at the last prompt position";
    ctx->poisoned = KIE_ERR_NONFINITE;
    return KIE_ERR_NONFINITE;
  }
  *next = tok;
  return KIE_OK;
}

extern "C" int kie_prefill_ex(kie_ctx *ctx, const int32_t *tokens, int32_t n, int32_t *next_token,
                              float *logits_out) {
  if (!ctx || !tokens || !next_token || n < 1) return KIE_ERR_INVALID;
  if (ctx->poisoned) return KIE_ERR_POISONED;
  if (n > ctx->m.max_seq) return KIE_ERR_CAPACITY;
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= ctx->m.vocab) return KIE_ERR_INVALID;
  CK(cudaMemsetAsync(ctx->kcache, 0xff, ctx->kv_elems * 2, ctx->stream));
  CK(cudaMemsetAsync(ctx->vcache, 0xff, ctx->kv_elems * 2, ctx->stream));
  ctx->pos = 0;
  ctx->pending = -1;
  int32_t next = -1;
  if (ctx->prefill_gemm) {
    if (int rc = prefill_gemm_run(ctx, tokens, n, logits_out, &next)) return rc;
  } else {
    std::vector<int32_t> out(n);
    if (int rc = run(ctx, 0, n, tokens, 0, false, logits_out, out.data())) return rc;
    ctx->last_prefill_ms = ctx->last_ms;
    next = out[n - 1];
  }
  ctx->pos = n;
  ctx->pending = next;
  *next_token = next;
  return KIE_OK;
}

extern "C" int kie_prefill(kie_ctx *ctx, const int32_t *tokens, int32_t n, int32_t *next_token) {
  return kie_prefill_ex(ctx, tokens, n, next_token, nullptr);
}

extern "C" int kie_set_prefill_mode(kie_ctx *ctx, int32_t mode) {
  if (!ctx || (mode != KIE_PREFILL_STEPS && mode != KIE_PREFILL_GEMM)) return KIE_ERR_INVALID;
  if (mode == KIE_PREFILL_GEMM && !ctx->prefill_gemm_ok) {
    g_last_error = "the tensor-core prompt pass is not available for this model (lane models, or no "
                   "device memory for its weight copy)";
    return KIE_ERR_INVALID;
  }
  ctx->prefill_gemm = mode == KIE_PREFILL_GEMM ? 1 : 0;
  return KIE_OK;
}

extern "C" int kie_decode_ex(kie_ctx *ctx, int32_t n_steps, const int32_t *forced_tokens,
                             int32_t *out_tokens, float *logits_out) {
  if (!ctx || !out_tokens || n_steps < 1) return KIE_ERR_INVALID;
  if (ctx->poisoned) return KIE_ERR_POISONED;
  if (!forced_tokens && ctx->pending < 0) return KIE_ERR_INVALID;
  if (int64_t(ctx->pos) + n_steps > ctx->m.max_seq) return KIE_ERR_CAPACITY;
  if (forced_tokens)
    for (int i = 0; i < n_steps; ++i)
      if (forced_tokens[i] < 0 || forced_tokens[i] >= ctx->m.vocab) return KIE_ERR_INVALID;
  int rc = run(ctx, ctx->pos, n_steps, forced_tokens, ctx->pending, true, logits_out, out_tokens);
  if (rc) return rc;
  ctx->pos += n_steps;
  ctx->pending = out_tokens[n_steps - 1];
  return KIE_OK;
}

extern "C" int kie_decode(kie_ctx *ctx, int32_t n_steps, int32_t *out_tokens) {
  return kie_decode_ex(ctx, n_steps, nullptr, out_tokens, nullptr);
}

extern "C" int kie_decode_sample(kie_ctx *ctx, int32_t n_steps, const kie_sampling *params,
                                 const float *uniforms, const int32_t *forced_tokens,
                                 int32_t *out_tokens, float *logits_out) {
  if (!ctx || !out_tokens || !params || n_steps < 1) return KIE_ERR_INVALID;
  if (ctx->poisoned) return KIE_ERR_POISONED;
  const float T = params->temperature;
  if (!(T >= 0.f) || !std::isfinite(T)) {
    g_last_error = "temperature must be finite and >= 0";
    return KIE_ERR_INVALID;
  }
  if (T == 0.f) return kie_decode_ex(ctx, n_steps, forced_tokens, out_tokens, logits_out);
  if (params->top_k < 0 || params->top_k > KIE_MAX_TOP_K || !(params->top_p > 0.f) ||
      !(params->top_p <= 1.f) || (params->top_k == 0 && params->top_p != 1.f)) {
    g_last_error = "top_k must lie in [0, KIE_MAX_TOP_K] and top_p in (0, 1], with top_p 1 when top_k is 0";
    return KIE_ERR_INVALID;
  }
  if (params->top_k > 0 && ctx->max_lm_rows > kMaxSampleRows) {
    g_last_error = "vocabulary slice per SM too large for a top-k cut";
    return KIE_ERR_INVALID;
  }
  if (params->top_k == 0 && ctx->plan.vbuf_floats < ctx->plan.n_ctas + 1) {
    g_last_error = "too many SMs for sampling without a top-k cut";
    return KIE_ERR_INVALID;
  }
  if (!uniforms) return KIE_ERR_INVALID;
  for (int i = 0; i < n_steps; ++i)
    if (!(uniforms[i] >= 0.f && uniforms[i] < 1.f)) {
      g_last_error = "uniforms must lie in [0, 1)";
      return KIE_ERR_INVALID;
    }
  if (!forced_tokens && ctx->pending < 0) return KIE_ERR_INVALID;
  if (int64_t(ctx->pos) + n_steps > ctx->m.max_seq) return KIE_ERR_CAPACITY;
  if (forced_tokens)
    for (int i = 0; i < n_steps; ++i)
      if (forced_tokens[i] < 0 || forced_tokens[i] >= ctx->m.vocab) return KIE_ERR_INVALID;
  int rc = run(ctx, ctx->pos, n_steps, forced_tokens, ctx->pending, true, logits_out, out_tokens,
               params, uniforms);
  if (rc) return rc;
  ctx->pos += n_steps;
  ctx->pending = out_tokens[n_steps - 1];
  return KIE_OK;
}

extern "C" int kie_destroy(kie_ctx *ctx) {
  if (!ctx) return KIE_ERR_INVALID;
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  free_ctx(ctx);
  return KIE_OK;
}

extern "C" const char *kie_strerror(int status) {
  static thread_local std::string msg;
  const char *base = "unknown status";
  switch (status) {
    case KIE_OK: base = "ok"; break;
    case KIE_ERR_INVALID: base = "invalid argument"; break;
    case KIE_ERR_OOM: base = "out of device memory"; break;
    case KIE_ERR_CUDA: base = "CUDA error"; break;
    case KIE_ERR_CAPACITY: base = "KV capacity exceeded"; break;
    case KIE_ERR_NOT_RESIDENT: base = "persistent grid cannot be co-resident"; break;
    case KIE_ERR_DEVICE_TIMEOUT: base = "device watchdog timeout"; break;
    case KIE_ERR_POISONED: base = "context poisoned by an earlier device error"; break;
    case KIE_ERR_NONFINITE: base = "non-finite logits on the device"; break;
  }
  msg = base;
  if (!g_last_error.empty() && status != KIE_OK) msg += ": " + g_last_error;
  return msg.c_str();
}

extern "C" int kie_get_stats(const kie_ctx *ctx, kie_stats *out) {
  if (!ctx || !out) return KIE_ERR_INVALID;
  const Plan &P = ctx->plan;
  memset(out, 0, sizeof *out);
  out->n_ctas = P.n_ctas;
  out->threads_per_cta = monokernel_threads();
  out->ring_slots = P.ring_slots;
  out->slot_bytes = kSlotBytes;
  out->smem_bytes = int32_t(P.smem);
  out->pos = ctx->pos;
  out->weight_bytes_per_step = P.weight_bytes_per_step;
  out->kv_bytes_per_position = int64_t(2) * ctx->m.n_layers * ctx->m.n_kv_heads * ctx->m.head_dim * 2;
  out->last_kernel_ms = ctx->last_ms;
  out->last_launch_steps = ctx->last_steps;
  out->pending_token = ctx->pending;
  out->last_prefill_ms = ctx->last_prefill_ms;
  out->prefill_mode = ctx->prefill_gemm ? KIE_PREFILL_GEMM : KIE_PREFILL_STEPS;
  return KIE_OK;
}

extern "C" int kie_copy_kv(const kie_ctx *ctx, int32_t layer, int32_t kv_head, int32_t pos0,
                           int32_t n, uint16_t *k_out, uint16_t *v_out) {
  if (!ctx) return KIE_ERR_INVALID;
  const kie_model_desc &m = ctx->m;
  if (layer < 0 || layer >= m.n_layers || kv_head < 0 || kv_head >= m.n_kv_heads || pos0 < 0 ||
      n < 0 || int64_t(pos0) + n > m.max_seq)
    return KIE_ERR_INVALID;
  const size_t off = ((size_t(layer) * m.n_kv_heads + kv_head) * m.max_seq + pos0) * m.head_dim;
  const size_t bytes = size_t(n) * m.head_dim * 2;
  kie_ctx *c = const_cast<kie_ctx *>(ctx);
  cudaError_t e = cudaSuccess;
  if (k_out && e == cudaSuccess) e = cudaMemcpyAsync(k_out, ctx->kcache + off, bytes, cudaMemcpyDeviceToHost, ctx->stream);
  if (v_out && e == cudaSuccess) e = cudaMemcpyAsync(v_out, ctx->vcache + off, bytes, cudaMemcpyDeviceToHost, ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  if (e != cudaSuccess) return cuda_fail(c, "kv copy", e);
  return KIE_OK;
}

extern "C" int kie_get_profile(const kie_ctx *ctx, uint64_t *out, int32_t n_words) {
  if (!ctx || !out) return KIE_ERR_INVALID;
  if (!monokernel_profiled()) {
    g_last_error = "not a profiling build";
    return KIE_ERR_INVALID;
  }
  const int32_t need = ctx->plan.n_ctas * kProfSlots;
  if (n_words < need) return KIE_ERR_INVALID;
  cudaError_t e = cudaMemcpy(out, ctx->prof, size_t(need) * 8, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(const_cast<kie_ctx *>(ctx), "profile copy", e);
  return KIE_OK;
}

extern "C" int kie_trace_request(kie_ctx *ctx, int32_t cta, int32_t step) {
  if (!ctx || cta < 0 || cta >= ctx->plan.n_ctas) return KIE_ERR_INVALID;
  if (!monokernel_profiled()) {
    g_last_error = "not a profiling build";
    return KIE_ERR_INVALID;
  }
  ctx->trace_cta = cta;
  ctx->trace_step = step;
  return KIE_OK;
}

extern "C" int kie_get_trace(const kie_ctx *ctx, uint64_t *out, int32_t n_words) {
  if (!ctx || !out || n_words < 1) return KIE_ERR_INVALID;
  if (!ctx->trace) {
    g_last_error = "not a profiling build";
    return KIE_ERR_INVALID;
  }
  const int32_t n = std::min<int32_t>(n_words, kTraceCap + 1);
  cudaError_t e = cudaMemcpy(out, ctx->trace, size_t(n) * 8, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(const_cast<kie_ctx *>(ctx), "trace copy", e);
  return KIE_OK;
}

extern "C" int kie_debug_set(kie_ctx *ctx, int32_t watchdog_ms, int32_t skip_signal_cta) {
  if (!ctx || watchdog_ms < 1) return KIE_ERR_INVALID;
  ctx->watchdog_ns = uint64_t(watchdog_ms) * 1000000ull;
  ctx->skip_signal_cta = skip_signal_cta;
  return KIE_OK;
}

extern "C" int kie_set_max_steps_per_launch(kie_ctx *ctx, int32_t n) {
  if (!ctx || n < 0) return KIE_ERR_INVALID;
  ctx->max_launch_steps = n;
  return KIE_OK;
}

extern "C" int kie_set_sum_mode(kie_ctx *ctx, int32_t mode) {
  if (!ctx || (mode != KIE_SUM_FP32_ATOMIC && mode != KIE_SUM_EXACT)) return KIE_ERR_INVALID;
  ctx->det_sum = mode == KIE_SUM_EXACT ? 1 : 0;
  return KIE_OK;
}

extern "C" int kie_set_sync_mode(kie_ctx *ctx, int32_t mode) {
  if (!ctx || (mode != KIE_SYNC_DEPENDENCY && mode != KIE_SYNC_GRID)) return KIE_ERR_INVALID;
  ctx->grid_sync = mode == KIE_SYNC_GRID ? 1 : 0;
  return KIE_OK;
}

// ---------------------------------------------------------------- decode without allocation
// kie_decode_ex_static: the same decode as kie_decode_ex, but the persistent
// kernel's per-launch scratch (activation vectors, attention partials, the
// epoch counters, argmax keys, token staging) lives in this fixed array that
// the library's device image carries, instead of in buffers of the context.
// The call itself makes no device or host allocation: it only copies, sets
// memory and launches.  One array per GPU, held from module load until the
// process exits; every call on that GPU reuses it.
namespace {
constexpr size_t kStaticScratchBytes = size_t(1) << 20;   // 1 MiB
constexpr int kStaticMaxDevices = 64;
}  // namespace
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
static void *g_static_scratch_dev[kStaticMaxDevices];
static std::mutex g_static_scratch_mu;

// Device address of g_static_scratch on `device` (the current device).  The
// symbol's name is only a host-side handle, so the address is looked up once
// per device with cudaGetSymbolAddress and cached.
static int static_scratch_address(int device, void **out) {
  if (device < 0 || device >= kStaticMaxDevices) {
    g_last_error = "device index beyond the static scratch table";
    return KIE_ERR_INVALID;
  }
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_dev[device]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      set_error("cudaGetSymbolAddress(static scratch)", e);
      return KIE_ERR_CUDA;
    }
    g_static_scratch_dev[device] = p;
  }
  *out = g_static_scratch_dev[device];
  return KIE_OK;
}

extern "C" int kie_decode_ex_static(kie_ctx *ctx, int32_t n_steps, const int32_t *forced_tokens,
                                    int32_t *out_tokens, float *logits_out) {
  if (!ctx || !out_tokens || n_steps < 1) return KIE_ERR_INVALID;
  if (ctx->poisoned) return KIE_ERR_POISONED;
  if (!forced_tokens && ctx->pending < 0) return KIE_ERR_INVALID;
  if (int64_t(ctx->pos) + n_steps > ctx->m.max_seq) return KIE_ERR_CAPACITY;
  if (forced_tokens)
    for (int i = 0; i < n_steps; ++i)
      if (forced_tokens[i] < 0 || forced_tokens[i] >= ctx->m.vocab) return KIE_ERR_INVALID;
  // carve the scratch: counters | keys | forced tokens | out tokens | activations
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t sync_bytes = size_t(SY_COUNT) * kSyncStride * 4;
  const size_t o_keys = up(sync_bytes);
  const size_t o_tin = o_keys + up(size_t(n_steps) * 8);
  const size_t o_tout = o_tin + up(size_t(n_steps) * 4);
  const size_t o_act = o_tout + up(size_t(n_steps) * 4);
  const size_t need = o_act + ctx->act_floats * 4;
  if (need > kStaticScratchBytes) {
    char buf[200];
    snprintf(buf, sizeof buf,
             "static scratch too small: this model and %d steps need %zu bytes, the fixed "
             "maximum is %zu",
             n_steps, need, kStaticScratchBytes);
    g_last_error = buf;
    return KIE_ERR_CAPACITY;
  }
  void *base = nullptr;
  int device = -1;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(ctx, "cudaGetDevice", e);
  if (device != ctx->device) {
    g_last_error = "the context's device is not the current device";
    return KIE_ERR_INVALID;
  }
  if (int rc = static_scratch_address(device, &base)) return rc;
  uint8_t *s = static_cast<uint8_t *>(base);
  float *act = reinterpret_cast<float *>(s + o_act);

  // Same arguments as kie_decode_ex (a pending kie_debug_set hook applies to
  // this call and is consumed by it), except that every per-launch buffer is
  // carved from the fixed array.  The profiling build's activity counters and
  // trace are not wired here: they live in buffers of the context.
  KernelArgs a = fill_args(ctx, ctx->pos, n_steps, ctx->pending, true, logits_out);
  set_act(ctx, a, act);
  a.sync = reinterpret_cast<uint32_t *>(s);
  a.keys = reinterpret_cast<unsigned long long *>(s + o_keys);
  a.forced = forced_tokens ? reinterpret_cast<const int32_t *>(s + o_tin) : nullptr;
  a.out_tokens = reinterpret_cast<int32_t *>(s + o_tout);

  if (forced_tokens)
    CK(cudaMemcpyAsync(s + o_tin, forced_tokens, size_t(n_steps) * 4, cudaMemcpyHostToDevice,
                       ctx->stream));
  if (int rc = launch_steps(ctx, a, sync_bytes, n_steps, out_tokens)) return rc;
  ctx->pos += n_steps;
  ctx->pending = out_tokens[n_steps - 1];
  return KIE_OK;
}
