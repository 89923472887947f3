// Host-only check of the decode kernel's plan (no GPU calls): for each shape,
// the repack copies every weight element into the per-SM streams exactly once;
// the tiles the producer issues and the consumers take agree; the row-stage
// mapping (row blocks of one input slice; in each column tile, lane l a row,
// warp w a run of 16-byte chunks stored at a position swizzled by the row) and
// the column-stage thread mapping cover every weight once and, emulated in
// double precision on the streamed bytes, reproduce the canonical
// matrix-vector products of one layer; the attention splits partition the
// positions; shared-memory budgets hold.  Built and run by tests/test_plan.py.
#include "../decode_persistent_monokernel_b200/csrc/kie_api.cu"
#include <random>

static int fails = 0;
#define REQ(c, ...) do { if (!(c)) { printf("FAIL %s:%d: ", __FILE__, __LINE__); printf(__VA_ARGS__); printf("\n"); if (++fails > 20) exit(1);} } while (0)

static void check(kie_model_desc m, int n_ctas, const char *name) {
  Plan P;
  const char *why = build_plan(m, n_ctas, 232448, P);
  if (why) { printf("%s: plan error %s\n", name, why); fails++; return; }
  const Layout Ly = make_layout(m);
  printf("%s: ctas %d slots %d smem %zu vbuf %d part %d stream %.3f GB jobs %zu blocks %zu\n", name, n_ctas,
         P.ring_slots, P.smem, P.vbuf_floats, P.part_floats, P.stream_bytes / 1e9, P.jobs.size(), P.blocks.size());
  REQ(P.smem <= 232448, "smem");
  for (int k = 0; k < ST_COUNT; ++k)
    printf("  stage %d: K %d R %d nseg %d norm %d cps %d cols %d\n", k, P.shape[k].K, P.shape[k].R,
           P.shape[k].nseg, P.shape[k].norm, P.shape[k].cps, P.shape[k].cols);
  const int nl = m.n_lanes, d = m.d_model, dh = m.head_dim, dl = d / nl, Hkv = m.n_kv_heads;
  const int hq = m.n_heads / nl, hkv = Hkv / nl, fl = m.ffn_dim / nl, G = m.n_heads / Hkv;
  const bool lanes = nl > 1;
  // ---- 1. repack coverage
  std::vector<uint8_t> seen(Ly.total, 0);
  std::mt19937 rng(7);
  std::vector<uint16_t> W(Ly.total);
  for (auto &w : W) w = uint16_t(rng() % 7);
  std::vector<uint16_t> S(P.stream_bytes / 2, 0xdead);
  for (const RepackJob &j : P.jobs) {
    REQ(j.dst_byte % 16 == 0 && j.K % 4 == 0, "align");
    if (j.trans == 2) {
      REQ(j.kb % 128 == 0 && j.K % j.kb == 0 && j.rb0 + j.nrows <= j.rb && j.rb <= kMaxRowBlock, "tiled job shape");
      REQ(j.dst_byte + int64_t(j.rb) * j.K * 2 <= P.stream_bytes, "dst range");
      REQ(j.src_elem % 8 == 0, "tiled job alignment");
    } else {
      REQ(j.dst_byte + int64_t(j.nrows) * j.K * 2 <= P.stream_bytes, "dst range");
    }
    for (int i = 0; i < j.nrows; ++i)
      for (int r = 0; r < j.K; ++r) {
        const int64_t src = j.trans == 1 ? j.src_elem + int64_t(r) * j.src_ld + i : j.src_elem + int64_t(i) * j.K + r;
        REQ(src >= 0 && src < Ly.total, "src range");
        if (seen[src]) { REQ(false, "copied twice %ld", (long)src); return; }
        seen[src] = 1;
        int64_t dst = j.dst_byte / 2 + int64_t(i) * j.K + r;
        if (j.trans == 2) {   // tile t = r / kb, chunk (r % kb) / 8 swizzled by the tile row
          const int t = r / j.kb, c = (r % j.kb) / 8, e = r % 8, tr = j.rb0 + i;
          dst = j.dst_byte / 2 + (int64_t(t) * j.rb + tr) * j.kb + int64_t(c ^ (tr & 7)) * 8 + e;
        }
        REQ(S[dst] == 0xdead, "dst written twice");
        S[dst] = W[src];
      }
    if (!j.trans) REQ(j.src_elem % 8 == 0, "plain job alignment");
  }
  int64_t uncopied = 0;
  for (int64_t i = 0; i < Ly.total; ++i) uncopied += !seen[i];
  const int64_t norms = int64_t(m.n_layers) * 2 * d + d;
  REQ(uncopied == int64_t(m.vocab) * d + norms, "uncopied %ld", (long)uncopied);

  // ---- 2. stage emulation for one layer (layer 1, or 0)
  const int layer = m.n_layers > 1 ? 1 : 0;
  const int64_t lay = Ly.layer0 + int64_t(layer) * Ly.layer_stride;
  auto lanep = [&](int ln) { return lay + int64_t(ln) * Ly.lane_stride; };
  auto vin = [&](int i) { return double(i % 5 + 1); };        // row-stage input
  auto oval = [&](int col) { return double(col % 7 + 1); };   // attention output (global o index)
  auto hval = [&](int j) { return double(j % 3 + 1); };       // hidden unit
  std::vector<double> qkv((m.n_heads + 2 * Hkv) * dh, 0.0);
  std::vector<int> qkv_hit(qkv.size(), 0);
  std::vector<double> accO(d, 0.0), accD(d, 0.0), hidden(m.ffn_dim, 0.0);
  std::vector<int> h_hit(m.ffn_dim, 0);
  for (int c = 0; c < n_ctas; ++c) {
    const int g = c % Hkv;
    int64_t cur = P.cta_stream_off[c] / 2;
    // walk stage instances in stream order until `layer`
    for (int l = 0; l <= layer; ++l) {
      const int seq[5] = {ST_QKV, ST_MIX, ST_O, ST_GU, ST_D};
      for (int k : seq) {
        if (k == ST_MIX && !(lanes && l >= 1)) continue;
        const StageCta &sc = P.stage_cta[size_t(k) * n_ctas + c];
        const StageShape &sh = P.shape[k];
        std::vector<int64_t> tstart;
        int t = 0;
        // the tiles the producer issues and the consumers take: every row
        // block's column tiles (row stages), R rows of each block (column stages)
        std::vector<Block> rbs, obs;
        for (int bi = 0; bi < sc.nblk; ++bi) obs.push_back(P.blocks[P.cta_blk_begin[c] + sc.blk_begin + bi]);
        if (!sh.cols)
          for (int bi = 0; bi < sc.nrb; ++bi) rbs.push_back(P.blocks[P.cta_blk_begin[c] + sc.rb_begin + bi]);
        if (!sh.cols) {
          const int kb = 128 * sh.cps, nk = sh.K / kb;
          REQ(sh.cps == 1 || sh.cps == 2 || sh.cps == 4, "cps");
          REQ(sh.R * sh.cps == kMaxRowBlock && sh.K % kb == 0, "row tiling");
          std::vector<int> cover(std::max(1, sc.nlocal), 0);
          for (const Block &b : rbs) {
            REQ(b.tile0 == t && b.nrows >= 1 && b.nrows <= sh.R, "row block");
            REQ(int64_t(b.nrows) * kb * 2 <= kSlotBytes, "row tile fits a slot");
            for (int i = 0; i < b.nrows; ++i) {
              REQ(b.lrow0 + i < sc.nlocal, "row block rows");
              cover[b.lrow0 + i]++;
              bool found = false;   // the row's output block reads the block's input slice
              for (const Block &o : obs)
                if (b.lrow0 + i >= o.lrow0 && b.lrow0 + i < o.lrow0 + o.nrows) { found = true; REQ(o.in_off == b.in_off, "one input slice"); }
              REQ(found, "row in an output block");
            }
            for (int q = 0; q < nk; ++q) {
              tstart.push_back(cur);
              cur += int64_t(b.nrows) * kb;
              ++t;
            }
          }
          for (int i = 0; i < sc.nlocal; ++i) REQ(cover[i] == 1, "row blocks cover local rows once");
        } else {
          for (const Block &b : obs) {
            REQ(b.tile0 == t, "tile0");
            for (int r0 = 0; r0 < b.nrows; r0 += sh.R) {
              const int rows = std::min(sh.R, b.nrows - r0);
              REQ(int64_t(rows) * sh.K * 2 <= kSlotBytes, "slot");
              tstart.push_back(cur);
              cur += int64_t(rows) * sh.K;
              ++t;
            }
          }
        }
        REQ(t == sc.ntiles, "ntiles");
        if (l != layer) continue;
        if (!sh.cols) {
          // row stage: lane / warp mapping of Consumer::gemv_rows_c
          const int C = sh.cps, kb = 128 * C, nk = sh.K / kb;
          std::vector<double> rowpart(size_t(std::max(1, sc.nlocal)) * kConsumerWarps, 0.0);
          std::vector<int> chunk_hit(size_t(std::max(1, sc.nlocal)) * (sh.K / 8), 0);
          for (const Block &b : rbs) {
            for (int tt = 0; tt < nk; ++tt) {
              const int64_t ts = tstart[b.tile0 + tt];
              for (int w = 0; w < kConsumerWarps; ++w)
                for (int lane = 0; lane < 32; ++lane)
                  for (int j = 0; j < 4 / C; ++j) {
                    const int r = lane + 32 * j;
                    if (r >= b.nrows) continue;
                    for (int cc = 0; cc < C; ++cc) {
                      const int pch = w * C + cc;                   // logical chunk of the tile row
                      const int off = r * kb + ((pch ^ (r & 7)) << 3);   // element offset in the tile
                      REQ(off % 8 == 0 && off + 8 <= b.nrows * kb, "tile offset");
                      REQ(off * 2 + 16 <= kSlotBytes, "smem");
                      const int col = tt * kb + pch * 8;           // canonical column
                      REQ(b.in_off + col + 8 <= sh.in_len, "input slice");
                      double dsum = 0;
                      for (int e = 0; e < 8; ++e) dsum += double(S[ts + off + e]) * vin(b.in_off + col + e);
                      const int lr = b.lrow0 + r;
                      rowpart[size_t(lr) * kConsumerWarps + w] += dsum;
                      chunk_hit[size_t(lr) * (sh.K / 8) + col / 8]++;
                    }
                  }
            }
            REQ(kConsumerWarps * kMaxRowBlock * 2 <= P.rsum_off, "partials region");
          }
          if (k != ST_LM) REQ(P.rsum_off + sc.nlocal <= P.part_floats, "row sums region");
          for (size_t q = 0; q < size_t(sc.nlocal) * (sh.K / 8); ++q) REQ(chunk_hit[q] == 1, "stage %d chunk hit %d", k, chunk_hit[q]);
          auto rowsum = [&](int i) { double v = 0; for (int w = 0; w < kConsumerWarps; ++w) v += rowpart[size_t(i) * kConsumerWarps + w]; return v; };
          if (k == ST_QKV) {
            for (int bi = 0; bi < sc.nblk; ++bi) {
              const Block &b = P.blocks[P.cta_blk_begin[c] + sc.blk_begin + bi];
              for (int i = 0; i < b.nrows; ++i) {
                const int o = b.out_off + i;
                REQ(o < (int)qkv.size(), "qkv index");
                qkv[o] = rowsum(b.lrow0 + i);
                qkv_hit[o]++;
                // which group owns row o
                const int qn = m.n_heads * dh;
                int owner = o < qn ? (o / dh) / G : (o < qn + Hkv * dh ? (o - qn) / dh : (o - qn - Hkv * dh) / dh);
                REQ(owner == g, "qkv row %d of group %d computed by group %d", o, owner, g);
              }
            }
          } else if (k == ST_GU) {
            for (int i = 0; i < sc.nout; ++i) {
              hidden[sc.row0 + i] = rowsum(i) * 1000.0 + rowsum(sc.nout + i);  // both halves checked
              h_hit[sc.row0 + i]++;
            }
          } else if (k == ST_MIX) {
            for (int i = 0; i < sc.nout; ++i) {
              const int r = sc.row0 + i;
              double want = 0;
              for (int kk = 0; kk < d; ++kk) want += double(W[Ly.layer0 + int64_t(layer - 1) * Ly.layer_stride + Ly.mix + int64_t(r) * d + kk]) * vin(kk);
              REQ(rowsum(i) == want, "mix row %d", r);
            }
          }
        } else {
          // column stage: thread mapping of Consumer::gemv_cols
          const int ngrp = sh.K / 4, tpr = sh.nseg > 1 ? ngrp : kConsumerWarps * 32;
          REQ((sh.R + sh.nseg - 1) / sh.nseg <= 8 / sh.cps && (sh.cps == 1 || sh.cps == 2), "rows per thread");
          std::vector<int> cover(size_t(ngrp) * 4096, 0);
          for (int bi = 0; bi < sc.nblk; ++bi) {
            const Block &b = P.blocks[P.cta_blk_begin[c] + sc.blk_begin + bi];
            const int ntile = (b.nrows + sh.R - 1) / sh.R;
            std::vector<double> out(sh.K, 0.0);
            std::vector<int> hit(size_t(b.nrows) * ngrp, 0);
            for (int tid = 0; tid < kConsumerWarps * 32; ++tid) {
              const int ph = tid / tpr, gi = tid - ph * tpr;
              if (ph >= sh.nseg) continue;
              for (int t = 0; t < ntile; ++t) {
                const int rows = std::min(sh.R, b.nrows - t * sh.R);
                for (int r = ph; r < rows; r += sh.nseg) {
                  const int li = b.lrow0 + t * sh.R + r;   // local scalar index
                  // scalar: O -> the group's attention output column; D -> hidden unit
                  double x;
                  if (k == ST_O) x = oval(G * g * dh + P.stage_cta[size_t(k) * n_ctas + c].row0 + li);
                  else x = hval(P.stage_cta[size_t(ST_GU) * n_ctas + c].row0 + li);
                  for (int j = 0; j < sh.cps; ++j) {
                    const int grp = gi + tpr * j;
                    REQ(grp < ngrp, "group");
                    const int64_t e = tstart[b.tile0 + t] + int64_t(r) * sh.K + int64_t(grp) * 4;
                    REQ((int64_t(r) * sh.K + grp * 4) * 2 + 8 <= kSlotBytes, "col smem");
                    for (int u = 0; u < 4; ++u) out[grp * 4 + u] += x * double(S[e + u]);
                    hit[size_t(t * sh.R + r) * ngrp + grp]++;
                  }
                }
              }
            }
            for (size_t q = 0; q < hit.size(); ++q) REQ(hit[q] == 1, "col cover");
            REQ(b.out_off + sh.K <= d, "out slice");
            for (int o = 0; o < sh.K; ++o) (k == ST_O ? accO : accD)[b.out_off + o] += out[o];
          }
          if (k == ST_O) REQ(sc.nlocal == sc.nout && sc.row0 + sc.nout <= G * dh, "o columns");
          if (k == ST_D) {
            const StageCta &gu = P.stage_cta[size_t(ST_GU) * n_ctas + c];
            REQ(gu.row0 == sc.row0 && gu.nout == sc.nout, "D slice = GU slice");
          }
        }
      }
    }
  }
  // ---- 3. compare the assembled vectors with canonical mat-vecs
  for (size_t o = 0; o < qkv.size(); ++o) {
    REQ(qkv_hit[o] == 1, "qkv row %zu hit %d", o, qkv_hit[o]);
    const int qn = m.n_heads * dh;
    int64_t src;
    int lnr;
    if ((int)o < qn) { const int h = o / dh; lnr = h / hq; src = lanep(lnr) + Ly.wq + int64_t(o - lnr * hq * dh) * dl; }
    else if ((int)o < qn + Hkv * dh) { const int r = o - qn, kv = r / dh; lnr = kv / hkv; src = lanep(lnr) + Ly.wk + int64_t(r - lnr * hkv * dh) * dl; }
    else { const int r = o - qn - Hkv * dh, kv = r / dh; lnr = kv / hkv; src = lanep(lnr) + Ly.wv + int64_t(r - lnr * hkv * dh) * dl; }
    double want = 0;
    for (int kk = 0; kk < dl; ++kk) want += double(W[src + kk]) * vin(lnr * dl + kk);
    REQ(qkv[o] == want, "qkv %zu got %f want %f", o, qkv[o], want);
  }
  for (int j = 0; j < m.ffn_dim; ++j) {
    REQ(h_hit[j] == 1, "hidden hit");
    const int ln = j / fl, jl = j % fl;
    double g0 = 0, u0 = 0;
    for (int kk = 0; kk < dl; ++kk) {
      g0 += double(W[lanep(ln) + Ly.wg + int64_t(jl) * dl + kk]) * vin(ln * dl + kk);
      u0 += double(W[lanep(ln) + Ly.wu + int64_t(jl) * dl + kk]) * vin(ln * dl + kk);
    }
    REQ(hidden[j] == g0 * 1000.0 + u0, "gate/up %d", j);
  }
  for (int r = 0; r < d; ++r) {
    const int ln = r / dl, rl = r % dl;
    double wo = 0, wd = 0;
    for (int col = 0; col < hq * dh; ++col) wo += double(W[lanep(ln) + Ly.wo + int64_t(rl) * hq * dh + col]) * oval(ln * hq * dh + col);
    for (int col = 0; col < fl; ++col) wd += double(W[lanep(ln) + Ly.wd + int64_t(rl) * fl + col]) * hval(ln * fl + col);
    REQ(accO[r] == wo, "O row %d got %f want %f", r, accO[r], wo);
    REQ(accD[r] == wd, "D row %d got %f want %f", r, accD[r], wd);
  }
  // ---- 4. LM tiles at the stream tail
  // ---- 5. attention splits partition [0, L) and the writer holds p
  for (int Lctx = 1; Lctx < 700; Lctx += 13)
    for (int gg = 0; gg < Hkv; ++gg) {
      const int nsplit = std::min((n_ctas - 1 - gg) / Hkv + 1, kMaxSplit);
      REQ(nsplit <= P.max_split, "max_split");
      int covered = 0;
      for (int c = gg; c < n_ctas; c += Hkv) {
        const int split = c / Hkv;
        if (split >= nsplit) continue;
        const int j0 = int((int64_t)split * Lctx / nsplit), j1 = int((int64_t)(split + 1) * Lctx / nsplit);
        REQ(j0 == covered, "partition");
        covered = j1;
        if (split == nsplit - 1) REQ(j0 <= Lctx - 1 && Lctx - 1 < j1, "writer");
      }
      REQ(covered == Lctx, "cover");
    }
  REQ((G + 2) * dh + kConsumerWarps * G * (dh + 2) <= P.vbuf_floats, "attn scratch");
  REQ(G * dh <= 512, "merged o");
  REQ(G * P.max_split * (dh + 2) <= P.vbuf_floats, "group partials in smem");
  for (int gg = 0; gg < Hkv; ++gg) {   // merge staging: (m, l) of every split + own columns
    const int ng = (n_ctas - 1 - gg) / Hkv + 1;
    for (int c = gg; c < n_ctas; c += Hkv) {
      const StageCta &so = P.stage_cta[size_t(ST_O) * n_ctas + c];
      REQ(2 * G * kMaxSplit + std::min(ng, kMaxSplit) * so.nout <= P.vbuf_floats, "merge staging");
    }
  }
  REQ(P.smem <= 232448 && P.ring_slots >= 3, "shared memory");
}

int main() {
  kie_model_desc c0{2, 256, 4, 4, 64, 704, 4096, 1e-5f, 1e4f, 0, 1, 0, 64};
  kie_model_desc gq{3, 256, 4, 2, 64, 704, 4096, 1e-5f, 1e4f, 0, 1, 0, 64};
  kie_model_desc g4{2, 256, 4, 1, 64, 704, 4096, 1e-5f, 1e4f, 0, 1, 0, 64};
  kie_model_desc l2{4, 256, 4, 4, 64, 704, 4096, 1e-5f, 1e4f, 0, 2, 2, 64};
  kie_model_desc l4{3, 1024, 8, 8, 128, 2048, 5000, 1e-5f, 1e4f, 0, 4, 3, 64};
  kie_model_desc d128{2, 512, 4, 2, 128, 1376, 5000, 1e-5f, 1e4f, 0, 1, 0, 64};
  kie_model_desc c1s{2, 2048, 16, 8, 128, 8192, 32768, 1e-5f, 1e4f, 0, 1, 0, 700};
  kie_model_desc c2s{3, 2048, 16, 16, 128, 8192, 32768, 1e-5f, 1e4f, 0, 8, 2, 700};
  kie_model_desc c4s{2, 4096, 32, 8, 128, 14336, 128256, 1e-5f, 5e5f, 1, 1, 0, 1300};
  check(c0, 148, "cfg0");
  check(gq, 148, "cfg0-gqa2");
  check(g4, 148, "cfg0-gqa4");
  check(c0, 20, "cfg0-20cta");
  // degenerate: fewer hidden units and vocabulary rows than SMs, so many SMs
  // have no gate/up/down rows and no LM-head rows; one query head per KV group
  kie_model_desc tinyv{2, 256, 4, 4, 64, 96, 100, 1e-5f, 1e4f, 0, 1, 0, 64};
  check(tinyv, 148, "degenerate-F96-V100");
  check(l2, 148, "lanes2");
  check(l4, 148, "lanes4");
  check(d128, 148, "dh128");
  check(c1s, 148, "cfg1-2L");
  check(c2s, 148, "cfg2-3L");
  check(c4s, 148, "cfg4-2L");
  for (auto [m, nm] : {std::pair{kie_model_desc{34, 2048, 16, 8, 128, 8192, 32768, 1e-5f, 1e4f, 0, 1, 0, 700}, "cfg1"},
                       std::pair{kie_model_desc{34, 2048, 16, 16, 128, 8192, 32768, 1e-5f, 1e4f, 0, 8, 2, 700}, "cfg2"},
                       std::pair{kie_model_desc{32, 4096, 32, 8, 128, 14336, 128256, 1e-5f, 5e5f, 1, 1, 0, 1300}, "cfg4"}}) {
    Plan P;
    const char *why = build_plan(m, 148, 232448, P);
    printf("%s: %s slots %d smem %zu stream %.3f GB wbytes %lld\n", nm, why ? why : "ok", P.ring_slots, P.smem,
           P.stream_bytes / 1e9, (long long)P.weight_bytes_per_step);
    // the named workloads run on shape-specialised kernel instances: their
    // model and plan must match an instance's key (else they would silently
    // fall back to the slower runtime-shape instance)
    const InstShape k = inst_shape(m, P), none{};
    if (m.n_lanes == 1) {
      REQ(monokernel_fn(m.dtype, 0, k) != monokernel_fn(m.dtype, 0, none), "%s: no shape-specialised dense instance", nm);
      REQ(monokernel_fn(m.dtype, 2, k) != monokernel_fn(m.dtype, 2, none), "%s: no shape-specialised sampling instance", nm);
    } else {
      REQ(monokernel_fn(m.dtype, 4, k) != monokernel_fn(m.dtype, 1, k), "%s: no lanes instance for its shape", nm);
    }
  }
  // row lengths: K / 128 lanes share a row, so only 128 x a power of two
  for (int K = 128; K <= 4096; K += 128) {
    StageShape sh;
    const bool pow2 = ((K >> 7) & ((K >> 7) - 1)) == 0;
    REQ((make_shape(K, K, K, K, sh) == nullptr) == pow2, "make_shape K=%d", K);
    if (pow2)
      for (int run = 1; run <= 300; run += 7) {   // every chunk width keeps a tile within a slot
        set_row_tiling(sh, run);
        REQ(128 * sh.cps <= K && K % (128 * sh.cps) == 0 && sh.R * sh.cps == kMaxRowBlock, "tiling K=%d", K);
        REQ(sh.R * 256 * sh.cps <= kSlotBytes, "tile bytes K=%d", K);
      }
  }
  {
    // a 3-lane model with 128-wide lanes: its d_model rows (mix, LM head)
    // have K = 384, which the plan must refuse
    Plan P;
    kie_model_desc m3{2, 384, 6, 3, 64, 768, 4096, 1e-5f, 1e4f, 0, 3, 2, 64};
    REQ(build_plan(m3, 148, 232448, P) != nullptr, "3-lane d_model 384 accepted");
  }
  {
    // which kernel instance each kind of call launches: the dense one unless an
    // ablation switch, the L2 look-ahead or a lane model needs another; the
    // sampler's when a temperature is set (lane models sample on the general one)
    struct Case { int lanes, grid, det, l2pf; float t; int want; };
    const Case cases[] = {{1, 0, 0, 0, 0.f, 0}, {1, 0, 0, 0, 0.7f, 2}, {8, 0, 0, 0, 0.f, 4},
                          {8, 0, 0, 0, 0.7f, 3}, {1, 1, 0, 0, 0.f, 1}, {1, 0, 1, 0, 0.f, 1},
                          {1, 0, 0, 4, 0.f, 1}, {1, 0, 1, 0, 0.7f, 3}, {8, 1, 0, 0, 0.f, 1}};
    for (const Case &c : cases) {
      KernelArgs a{};
      a.n_lanes = c.lanes; a.grid_sync = c.grid; a.det_sum = c.det; a.l2pf_tiles = c.l2pf; a.sample_t = c.t;
      REQ(kernel_variant(a) == c.want, "kernel_variant(lanes %d grid %d det %d l2pf %d T %g) = %d, want %d",
          c.lanes, c.grid, c.det, c.l2pf, c.t, kernel_variant(a), c.want);
    }
  }
  printf(fails ? "FAILED (%d)\n" : "ALL OK\n", fails);
  return fails != 0;
}
