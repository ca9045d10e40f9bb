// pa_plan.cpp — host planner: split count and workspace for one piece.
//
// splash PR #33 ("What changed") picks the split count from the GPU's core count, the KV
// heads and the piece's tiles, so that short pieces at long history still fill the GPU, and
// sizes the split workspace from it. On B200 one CTA of the prefill kernel owns one SM (it
// uses ~225 KB of shared memory and the whole 512-column tensor memory), so the question is
// how the (KV head, Q tile, split) units pack onto 148 SMs. The default policy answers it by
// simulating the launch: units are dispatched in index order (longest first) to the SM that
// frees first, and the split count with the smallest simulated makespan plus combine cost
// wins. The pages' own rule and the earlier rule it replaced are kept as policies.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <vector>

#include "pa.h"
#include "pa_geometry.h"
#include "pa_schedule.h"

namespace {

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Cost model (microseconds), B200, fitted to the kernels' measured cycle counts (regression
// over items of 4-256 tiles at ~1.7 GHz, head dim 256): a 128x128 KV tile costs 4*128*128*D
// FLOPs at about 1.5 PFLOP/s shared by 148 SMs; a unit pays a fixed start/finish cost (set-up,
// Q tile load and pipeline fill, writing 128 rows of fp32 output: ~13,000 cycles at D = 256);
// the combine streams the partials through HBM.
struct CostModel {
  double tile_us, unit_us, combine_us_per_byte, combine_fixed_us;
  explicit CostModel(int D) {
    const double per_sm_flops = 1.5e15 / 148.0;
    tile_us = 4.0 * pa::kTileKeys * pa::kTileRows * D / per_sm_flops * 1e6;
    unit_us = 3.0 + pa::kTileRows * (double)D * 4.0 / 30e9 * 1e6;
    combine_us_per_byte = 1.0 / 5.0e12 * 1e6;
    combine_fixed_us = 4.0;
  }
};

// K/V bytes of a piece above which the row blocks of a head are scheduled as teams (about
// three quarters of the 126 MB L2).
constexpr double kTeamKvBytes = 96e6;

// CTAs per unit: head dim 256 runs on CTA pairs (two Q tiles share each K/V tile load).
int ctas_per_unit_for(int D) { return D == 256 ? 2 : 1; }

double simulate(int num_sms, int64_t q_tiles, int64_t R, int G, int Hkv, int64_t H, int S,
                int D) {
  const CostModel cm(D);
  const int per = ctas_per_unit_for(D);
  const int64_t q_units = (q_tiles + per - 1) / per;
  std::priority_queue<double, std::vector<double>, std::greater<double>> sms;
  for (int i = 0; i < num_sms / per; ++i) sms.push(0.0);  // a pair unit holds two SMs
  double makespan = 0.0;
  // Units in launch order: last Q tile first; within a tile, KV heads then splits.
  for (int64_t qt = q_units - 1; qt >= 0; --qt) {
    const int64_t n_kt = pa::unit_kv_tiles(qt, per, q_tiles, R, G, H);
    for (int g = 0; g < Hkv; ++g) {
      for (int s = 0; s < S; ++s) {
        int64_t kt0, kt1;
        pa::split_range(n_kt, s, S, &kt0, &kt1);
        const double w = (kt1 - kt0) * cm.tile_us + cm.unit_us;
        const double t = sms.top() + w;
        sms.pop();
        sms.push(t);
        makespan = std::max(makespan, t);
      }
    }
  }
  (void)G;
  return makespan;
}

double combine_cost(int S, int64_t R, int Hq, int D) {
  if (S <= 1) return 0.0;
  const CostModel cm(D);
  const double bytes = (double)S * R * Hq * (D + 1) * 4.0 + (double)R * Hq * D * 4.0;
  return bytes * cm.combine_us_per_byte + cm.combine_fixed_us;
}

// Greedy dispatch of items, in order, to `slots` identical workers (what the hardware does
// with a grid of CTAs that each hold a whole SM or SM pair).
double simulate_items(const std::vector<pa::PaItem>& items, int slots, const CostModel& cm) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> q;
  for (int i = 0; i < slots; ++i) q.push(0.0);
  double makespan = 0.0;
  for (const pa::PaItem& it : items) {
    const double t = q.top() + (it.kt1 - it.kt0) * cm.tile_us + cm.unit_us;
    q.pop();
    q.push(t);
    makespan = std::max(makespan, t);
  }
  return makespan;
}

}  // namespace

namespace pa {

// McNaughton's wrap-around rule: lay the runs of KV tiles (lengths len[order[0]], ...) end to
// end, fill `workers` to an equal load in turn, and cut a run where a worker's share ends.
// Every worker then carries the same load and at most one cut per worker boundary is made; no
// piece shorter than `m` tiles is cut off, and no run is cut into more parts than the combine
// merges. Returns the pieces (run, first tile, end tile, worker, planned start).
struct Piece {
  int32_t rb, kt0, kt1, worker;
  double start;
};

static bool wrap_cut(const std::vector<int64_t>& len, const std::vector<int32_t>& order,
                     int workers, double c_item, std::vector<Piece>* out) {
  const int64_t n = (int64_t)order.size();
  if (n == 0 || workers <= 0) return false;
  double total = 0.0;
  int64_t max_len = 0;
  for (int32_t r : order) {
    total += (double)len[r];
    max_len = std::max(max_len, len[r]);
  }
  std::vector<Piece>& pieces = *out;
  // Wrap-around assignment for a given share per worker; returns the workers it needs.
  auto assign = [&](double share, int64_t m, double over) -> int {
    pieces.clear();
    int k = 0;
    double load = 0.0;
    for (int32_t rb : order) {
      int64_t o = 0, r = len[rb];
      while (r > 0) {
        const double room = share - load - c_item;
        int64_t take;
        if ((double)r <= room + over) {
          take = r;  // the rest fits (a little over is fine)
        } else if (load > 0.0 && room < (double)m) {
          ++k;       // this worker is full
          load = 0.0;
          if (k > workers) return k + 1;  // cannot fit: stop early
          continue;
        } else {
          // at least m tiles (a fresh worker always makes progress), and leave at least m
          take = std::max<int64_t>((int64_t)room, m);
          if (r - take < m) take = r;
        }
        pieces.push_back({rb, (int32_t)o, (int32_t)(o + take), k, load});
        load += (double)take + c_item;
        o += take;
        r -= take;
        if (r > 0) {
          ++k;
          load = 0.0;
        }
      }
    }
    return k + 1;
  };
  // The smallest share (from the even split of the tiles plus one item cost per run and per
  // cut) whose assignment fits the workers; no run in more parts than the combine merges (a
  // part may also start and end a worker part-way, hence one part of slack).
  double share = (total + c_item * (double)(n + workers - 1)) / workers;
  share = std::max(share, (double)max_len / (PA_MAX_SPLITS - 2) + c_item + 1.0);
  const int64_t m = std::max<int64_t>(4, (int64_t)(share / 32.0));
  const double over = 1.0 + share / 128.0;
  for (int it = 0; it < 400 && assign(share, m, over) > workers; ++it) share *= 1.002;
  return assign(share, m, over) <= workers;
}

// The schedule of a set of pieces of the row blocks (numbered 0 .. n_rb-1): workspace slots
// for the parts of cut row blocks, items in the order of their planned start (so that the
// hardware's first-free dispatch reproduces the plan), and the simulated makespan.
static bool finish_schedule(const std::vector<Piece>& pieces, int64_t n_rb, int slots, int per,
                            int head_dim, Schedule* out) {
  const CostModel cm(head_dim);
  if ((int64_t)pieces.size() > kMaxItems) return false;
  // workspace slots: consecutive for the parts of each cut row block, in row-block order
  std::vector<int32_t> parts(n_rb, 0);
  for (const Piece& pc : pieces) ++parts[pc.rb];
  std::vector<int32_t> first(n_rb, -1);
  Schedule sch;
  sch.rows_per_block = per * kTileRows;
  for (int64_t rb = 0; rb < n_rb; ++rb) {
    if (parts[rb] > 1) {
      first[rb] = sch.n_slots;
      sch.split.push_back({(int32_t)rb, sch.n_slots, parts[rb], 0});
      sch.n_slots += parts[rb];
    }
    sch.max_parts = std::max(sch.max_parts, parts[rb]);
  }
  if ((int64_t)sch.split.size() > kMaxSplitBlocks || sch.max_parts > PA_MAX_SPLITS) return false;
  // the parts of a row block take its slots in key order
  std::vector<const Piece*> by_key;
  for (const Piece& pc : pieces) by_key.push_back(&pc);
  std::stable_sort(by_key.begin(), by_key.end(), [](const Piece* x, const Piece* y) {
    return x->rb != y->rb ? x->rb < y->rb : x->kt0 < y->kt0;
  });
  std::vector<int32_t> slot_of(pieces.size(), -1);
  std::vector<int32_t> seen(n_rb, 0);
  for (const Piece* pc : by_key)
    if (parts[pc->rb] > 1) slot_of[pc - pieces.data()] = first[pc->rb] + seen[pc->rb]++;
  std::vector<std::pair<std::pair<double, int>, PaItem>> items;
  for (size_t i = 0; i < pieces.size(); ++i) {
    const Piece& pc = pieces[i];
    items.push_back({{pc.start, pc.worker}, PaItem{pc.rb, pc.kt0, pc.kt1, slot_of[i]}});
  }
  std::stable_sort(items.begin(), items.end(),
                   [](const auto& x, const auto& y) { return x.first < y.first; });
  for (const auto& o : items) sch.items.push_back(o.second);
  double comb = 0.0;
  if (!sch.split.empty()) {
    double bytes = 0.0;
    for (const PaSplitBlock& b : sch.split)
      bytes += (double)(b.nparts + 1) * sch.rows_per_block * (head_dim + 1) * 4.0;
    comb = bytes * cm.combine_us_per_byte + cm.combine_fixed_us;
  }
  sch.makespan_us = simulate_items(sch.items, slots, cm) + comb;
  *out = std::move(sch);
  return true;
}

// The wrap-around rule over whole row blocks, one worker (SM or SM pair) each.
static bool wrap_around(const std::vector<int64_t>& len, const std::vector<int32_t>& order,
                        int slots, int per, int head_dim, Schedule* out) {
  const CostModel cm(head_dim);
  const int64_t n_rb = (int64_t)len.size();
  if (n_rb > kMaxItems || n_rb == 0) return false;
  std::vector<Piece> pieces;
  if (!wrap_cut(len, order, slots, cm.unit_us / cm.tile_us, &pieces)) return false;
  return finish_schedule(pieces, n_rb, slots, per, head_dim, out);
}

// The wrap-around rule over teams: `bundles` are groups of row blocks that read the same KV
// head (longest first within a group); a team of t = bundle size workers runs a bundle piece
// [a, b) as one item per row block, all starting together, so the team streams each K/V tile
// of the head at the same time and L2 serves its repeated reads. `slots` / t teams; a bundle's
// length is its longest row block's, and shorter ones end their last piece early.
static bool wrap_teams(const std::vector<int64_t>& len,
                       const std::vector<std::vector<int32_t>>& bundles, int t, int slots,
                       int per, int head_dim, Schedule* out) {
  const CostModel cm(head_dim);
  const int64_t n_rb = (int64_t)len.size();
  const int teams = slots / t;
  if (teams < 1 || bundles.empty()) return false;
  std::vector<int64_t> blen(bundles.size());
  std::vector<int32_t> border(bundles.size());
  for (size_t b = 0; b < bundles.size(); ++b) {
    int64_t mx = 0;
    for (int32_t rb : bundles[b]) mx = std::max(mx, len[rb]);
    blen[b] = mx;
    border[b] = (int32_t)b;
  }
  std::vector<Piece> team_pieces;
  if (!wrap_cut(blen, border, teams, cm.unit_us / cm.tile_us, &team_pieces)) return false;
  std::vector<Piece> pieces;
  for (const Piece& tp : team_pieces) {
    const std::vector<int32_t>& members = bundles[tp.rb];
    for (size_t i = 0; i < members.size(); ++i) {
      const int32_t rb = members[i];
      if (tp.kt0 >= len[rb]) continue;
      pieces.push_back({rb, tp.kt0, (int32_t)std::min<int64_t>(tp.kt1, len[rb]),
                        tp.worker * t + (int32_t)i, tp.start});
    }
  }
  return finish_schedule(pieces, n_rb, slots, per, head_dim, out);
}

// The balanced schedule of one piece (R rows at history H) of q_units row blocks a KV head.
static bool balanced_piece(int64_t q_tiles, int64_t R, int64_t H, int G, int Hkv, int head_dim,
                           int num_sms, Schedule* out) {
  const int per = ctas_per_unit_for(head_dim);
  const int slots = std::max(1, num_sms / per);
  const int64_t q_units = (q_tiles + per - 1) / per;
  const int64_t n_rb = q_units * Hkv;
  if (n_rb > kMaxItems || n_rb <= 0) return false;
  std::vector<int64_t> len(n_rb);
  std::vector<int32_t> order;
  order.reserve(n_rb);
  for (int64_t rb = 0; rb < n_rb; ++rb) {
    int64_t qu;
    int g;
    rb_coords((int32_t)rb, q_units, Hkv, &qu, &g);
    len[rb] = unit_kv_tiles(qu, per, q_tiles, R, G, H);
  }
  // The row blocks of one KV head one after another, longest first within the head (which
  // the numbering rb = g, g + Hkv, ... already is).
  for (int g = 0; g < Hkv; ++g)
    for (int64_t rb = g; rb < n_rb; rb += Hkv) order.push_back((int32_t)rb);
  // When the piece's K/V do not fit in L2, every row block of a head reads all of the head's
  // keys from HBM unless the row blocks stream them together: measured on a 128-row piece at
  // 131,072 keys (3 row blocks a head) 3.0x the K/V bytes from HBM, and on a 512-row piece at
  // 34K keys (12 a head) 10x. Then the row blocks of a head run as teams (wrap_teams) of t
  // workers, t as large as leaves at most a tenth of the workers idle.
  const double kv_bytes = 2.0 * (double)(H + R) * Hkv * head_dim * 2.0;
  const int64_t k = q_units;  // row blocks a head
  if (kv_bytes > kTeamKvBytes && k >= 2) {
    for (int64_t r = 1; r <= k; ++r) {
      const int t = (int)ceil_div64(k, r);
      const int teams = slots / t;
      if (teams < 1 || slots - teams * t > slots / 10) continue;
      std::vector<std::vector<int32_t>> bundles;
      for (int g = 0; g < Hkv; ++g)
        for (int64_t i = 0; i < k; i += t) {
          std::vector<int32_t> b;
          for (int64_t j = i; j < std::min<int64_t>(k, i + t); ++j)
            b.push_back((int32_t)(g + j * Hkv));
          bundles.push_back(std::move(b));
        }
      if (wrap_teams(len, bundles, t, slots, per, head_dim, out)) return true;
      break;
    }
  }
  return wrap_around(len, order, slots, per, head_dim, out);
}

bool build_balanced(const pa_plan_t& p, Schedule* out) {
  return balanced_piece(p.q_tiles, p.chunk_rows, p.hist_len, p.group, p.n_kv_heads, p.head_dim,
                        p.num_sms, out);
}

int describe_batch(int batch, const int32_t* q_lens, const int64_t* hist_lens, int G, int Hkv,
                   int per, Batch* out) {
  if (batch <= 0 || !q_lens || !hist_lens || G <= 0 || Hkv <= 0) return PA_ERR_INVALID_ARG;
  if (batch > kMaxSeqs) return PA_ERR_UNSUPPORTED;
  Batch bt;
  for (int b = 0; b < batch; ++b) {
    const int64_t r = q_lens[b], h = hist_lens[b];
    if (r < 0 || h < 0) return PA_ERR_INVALID_ARG;
    if (h + r + kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    const int64_t q_units = ceil_div64(q_tiles_for(r, G), per);
    bt.seq.push_back({(int32_t)bt.total_rows, (int32_t)r, (int32_t)h, (int32_t)bt.row_blocks});
    bt.total_rows += r;
    bt.row_blocks += q_units * Hkv;
    bt.max_hist = std::max(bt.max_hist, h);
    if (bt.total_rows >= (int64_t(1) << 31) || bt.row_blocks > kMaxItems)
      return PA_ERR_UNSUPPORTED;
  }
  if (bt.total_rows == 0) return PA_ERR_INVALID_ARG;
  *out = std::move(bt);
  return PA_OK;
}

int batch_ctas_per_unit(int head_dim, int G, int batch, const int32_t* q_lens) {
  int64_t max_qt = 0;
  for (int b = 0; b < batch; ++b) max_qt = std::max(max_qt, q_tiles_for(q_lens[b], G));
  return head_dim == 256 && max_qt > 1 ? 2 : 1;
}

bool build_batch(int num_sms, int head_dim, int per, int G, int Hkv, const Batch& bt,
                 Schedule* out) {
  // One-row batches on the swapped decode kernel: two CTA slots per SM.
  if (batch_decode_swapped(head_dim, G, per, bt.seq.data(), (int)bt.seq.size()))
    num_sms *= kDecCtasPerSm;
  // one sequence: the single piece's schedule (row blocks numbered the same way)
  if (bt.seq.size() == 1 && per == ctas_per_unit_for(head_dim))
    return balanced_piece(q_tiles_for(bt.seq[0].rows, G), bt.seq[0].rows, bt.seq[0].hist, G,
                          Hkv, head_dim, num_sms, out);
  const int slots = std::max(1, num_sms / per);
  std::vector<int64_t> len;
  for (const PaSeq& sq : bt.seq) {
    const int64_t q_tiles = q_tiles_for(sq.rows, G);
    const int64_t q_units = ceil_div64(q_tiles, per);
    for (int64_t local = 0; local < q_units * Hkv; ++local) {
      int64_t qu;
      int g;
      rb_coords((int32_t)local, q_units, Hkv, &qu, &g);
      len.push_back(unit_kv_tiles(qu, per, q_tiles, sq.rows, G, sq.hist));
    }
  }
  std::vector<int32_t> order(len.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = (int32_t)i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t x, int32_t y) { return len[x] > len[y]; });
  if (wrap_around(len, order, slots, per, head_dim, out)) return true;
  // Too many row blocks to also cut some (the item table holds 512): every row block whole,
  // longest first, as the hardware's first-free dispatch then runs them (LPT order).
  if (len.size() > (size_t)kMaxItems || len.empty()) return false;
  const CostModel cm(head_dim);
  Schedule sch;
  sch.rows_per_block = per * kTileRows;
  for (int32_t rb : order) sch.items.push_back(PaItem{rb, 0, (int32_t)len[rb], -1});
  sch.makespan_us = simulate_items(sch.items, slots, cm);
  *out = std::move(sch);
  return true;
}

}  // namespace pa

extern "C" int pa_batch_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim,
                             int page_size, int batch, const int32_t* q_lens,
                             const int64_t* hist_lens, int dtype, float scale, pa_plan_t* plan) {
  if (!plan) return PA_ERR_INVALID_ARG;
  memset(plan, 0, sizeof *plan);
  if (num_sms <= 0 || n_q_heads <= 0 || n_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || isinf(scale)) return PA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (!is_pow2(page_size) || page_size < 16 || page_size > 128) return PA_ERR_UNSUPPORTED;
  const int G = n_q_heads / n_kv_heads;
  if (batch <= 0 || !q_lens || !hist_lens) return PA_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b)
    if (q_lens[b] < 0) return PA_ERR_INVALID_ARG;
  // CTA pairs only when some sequence has two Q tiles to pair; else one CTA per row block
  const int per = pa::batch_ctas_per_unit(head_dim, G, batch, q_lens);
  pa::Batch bt;
  const int st = pa::describe_batch(batch, q_lens, hist_lens, G, n_kv_heads, per, &bt);
  if (st != PA_OK) return st;
  pa::Schedule sch;
  if (!pa::build_batch(num_sms, head_dim, per, G, n_kv_heads, bt, &sch))
    return PA_ERR_UNSUPPORTED;
  int64_t q_tiles = 0;
  for (const pa::PaSeq& sq : bt.seq) q_tiles += pa::q_tiles_for(sq.rows, G);
  plan->num_sms = num_sms;
  plan->n_q_heads = n_q_heads;
  plan->n_kv_heads = n_kv_heads;
  plan->head_dim = head_dim;
  plan->page_size = page_size;
  plan->group = G;
  plan->chunk_rows = (int32_t)bt.total_rows;
  plan->q_tiles = (int32_t)q_tiles;
  plan->splits = sch.max_parts;
  plan->paged = 1;
  plan->dtype = dtype;
  plan->policy = PA_POLICY_BALANCED;
  plan->ctas_per_unit = per;
  plan->batch = batch;
  plan->hist_len = bt.max_hist;
  plan->units = (int64_t)sch.items.size();
  plan->scale = scale > 0.0f ? scale : (float)(1.0 / sqrt((double)head_dim));
  plan->est_us = (float)sch.makespan_us;
  plan->ws_bytes = (uint64_t)sch.n_slots * sch.rows_per_block * (head_dim + 1) * 4ull;
  return PA_OK;
}

extern "C" int pa_decode_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim,
                              int page_size, int batch, int64_t max_seq_len, int dtype,
                              float scale, int splits_override, pa_plan_t* plan) {
  if (!plan) return PA_ERR_INVALID_ARG;
  memset(plan, 0, sizeof *plan);
  if (num_sms <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || batch <= 0 || max_seq_len < 1)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (splits_override < 0 || !(scale >= 0.0f) || isinf(scale)) return PA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (!is_pow2(page_size) || page_size < 16 || page_size > 128) return PA_ERR_UNSUPPORTED;
  if (splits_override > PA_MAX_SPLITS) return PA_ERR_UNSUPPORTED;
  const int G = n_q_heads / n_kv_heads;
  if (G > pa::kTileRows) return PA_ERR_UNSUPPORTED;
  if (max_seq_len + pa::kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  const int64_t max_tiles = pa::ceil_div64(max_seq_len, pa::kTileKeys);
  int S = splits_override;
  if (S == 0) {  // about two units per CTA slot (two slots per SM for the swapped kernel)
    const int64_t slots =
        (int64_t)num_sms * (pa::decode_swapped(head_dim, G) ? pa::kDecCtasPerSm : 1);
    const int64_t want = pa::ceil_div64(2 * slots, (int64_t)batch * n_kv_heads);
    S = (int)std::max<int64_t>(1, std::min<int64_t>({want, (int64_t)PA_MAX_SPLITS, max_tiles}));
  }
  if ((int64_t)batch * n_kv_heads * S >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  const CostModel cm(head_dim);
  plan->num_sms = num_sms;
  plan->n_q_heads = n_q_heads;
  plan->n_kv_heads = n_kv_heads;
  plan->head_dim = head_dim;
  plan->page_size = page_size;
  plan->group = G;
  plan->chunk_rows = batch;
  plan->q_tiles = 1;
  plan->splits = S;
  plan->paged = 1;
  plan->dtype = dtype;
  plan->policy = splits_override > 0 ? -1 : PA_POLICY_MAKESPAN;
  plan->ctas_per_unit = 1;
  plan->batch = batch;
  plan->hist_len = max_seq_len;
  plan->units = (int64_t)batch * n_kv_heads * S;
  plan->scale = scale > 0.0f ? scale : (float)(1.0 / sqrt((double)head_dim));
  const double waves = std::ceil((double)plan->units / num_sms);
  plan->est_us = (float)(waves * (cm.unit_us + (double)max_tiles / S * cm.tile_us));
  plan->ws_bytes = S > 1 ? (uint64_t)S * batch * n_q_heads * (head_dim + 1) * 4ull : 0ull;
  return PA_OK;
}

extern "C" int pa_pieces(int chunk_rows, int64_t hist_len, int log2_budget, int32_t* rows_out,
                         int cap) {
  if (chunk_rows < 0 || hist_len < 0 || log2_budget < 1 || log2_budget > 62 || cap < 0)
    return PA_ERR_INVALID_ARG;
  const int64_t budget = int64_t(1) << log2_budget;
  int n = 0;
  int64_t h = hist_len, left = chunk_rows;
  while (left > 0) {
    // the largest power of two r <= left with r * (h + r) <= budget (at least one row)
    int64_t r = 1;
    while (2 * r <= left && 2 * r * (h + 2 * r) <= budget) r *= 2;
    if (rows_out && n < cap) rows_out[n] = (int32_t)r;
    ++n;
    h += r;
    left -= r;
  }
  return n;
}

extern "C" int pa_cores_policy_splits(int cores, int kv_heads, int tiles) {
  if (cores <= 0 || kv_heads <= 0 || tiles <= 0) return 1;
  const int target = std::min(256, std::max(32, (32 * cores) / kv_heads));
  return std::min(32, std::max(1, target / tiles));
}

extern "C" int pa_legacy_policy_splits(int kv_heads, int tiles) {
  if (kv_heads <= 0 || tiles <= 0) return 1;
  return std::min(32, std::max(1, 32 / (tiles * kv_heads)));
}

extern "C" int pa_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim, int page_size,
                       int chunk_rows, int64_t hist_len, int dtype, float scale,
                       int splits_override, int policy, int paged, pa_plan_t* plan) {
  if (!plan) return PA_ERR_INVALID_ARG;
  memset(plan, 0, sizeof *plan);
  if (num_sms <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || chunk_rows <= 0 || hist_len < 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (splits_override < 0 || policy < 0 || policy > PA_POLICY_BALANCED) return PA_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || isinf(scale)) return PA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (paged && (!is_pow2(page_size) || page_size < 16 || page_size > 128))
    return PA_ERR_UNSUPPORTED;
  if (splits_override > PA_MAX_SPLITS) return PA_ERR_UNSUPPORTED;
  // Tensor-map coordinates are 32-bit: keep every key row index (plus a tile) below 2^31.
  const int64_t total_keys = hist_len + chunk_rows;
  if (total_keys + pa::kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;

  const int G = n_q_heads / n_kv_heads;
  const int64_t q_tiles = pa::q_tiles_for(chunk_rows, G);
  if (q_tiles * n_kv_heads * PA_MAX_SPLITS * 2 >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  const int64_t max_kt = pa::tile_kv_tiles(q_tiles - 1, chunk_rows, G, hist_len);
  const int per = ctas_per_unit_for(head_dim);
  const int64_t q_units = (q_tiles + per - 1) / per;

  int S = 1;
  int used_policy = policy == PA_POLICY_BALANCED ? PA_POLICY_MAKESPAN : policy;
  if (splits_override > 0) {
    S = splits_override;
    used_policy = -1;
  } else if (policy == PA_POLICY_CORES) {
    S = pa_cores_policy_splits(num_sms, n_kv_heads, (int)std::min<int64_t>(q_tiles, 1 << 30));
  } else if (policy == PA_POLICY_LEGACY) {
    S = pa_legacy_policy_splits(n_kv_heads, (int)std::min<int64_t>(q_tiles, 1 << 30));
  } else {  // makespan, and the uniform candidate of the balanced policy
    double best = 0.0;
    const int64_t base_units = q_units * n_kv_heads;
    for (int cand = 1; cand <= PA_MAX_SPLITS; ++cand) {
      if (cand > 1 && cand > max_kt) break;                   // more splits than KV tiles
      if (cand > 1 && base_units * per * cand > 16LL * num_sms) break;  // far past full
      const double t = simulate(num_sms, q_tiles, chunk_rows, G, n_kv_heads, hist_len, cand,
                                head_dim) +
                       combine_cost(cand, chunk_rows, n_q_heads, head_dim);
      if (cand == 1 || t < best * 0.98) {  // a new split must win by 2% to be worth it
        best = t;
        S = cand;
      }
    }
  }

  plan->num_sms = num_sms;
  plan->n_q_heads = n_q_heads;
  plan->n_kv_heads = n_kv_heads;
  plan->head_dim = head_dim;
  plan->page_size = paged ? page_size : 0;
  plan->group = G;
  plan->chunk_rows = chunk_rows;
  plan->q_tiles = (int32_t)q_tiles;
  plan->splits = S;
  plan->paged = paged ? 1 : 0;
  plan->dtype = dtype;
  plan->policy = used_policy;
  plan->ctas_per_unit = per;
  plan->batch = 0;
  plan->hist_len = hist_len;
  plan->units = q_units * n_kv_heads * S;
  plan->scale = scale > 0.0f ? scale : (float)(1.0 / sqrt((double)head_dim));
  plan->est_us = (float)(simulate(num_sms, q_tiles, chunk_rows, G, n_kv_heads, hist_len, S,
                                  head_dim) +
                         combine_cost(S, chunk_rows, n_q_heads, head_dim));
  plan->ws_bytes = S > 1 ? (uint64_t)S * chunk_rows * n_q_heads * (head_dim + 1) * 4ull : 0ull;

  // The balanced schedule: always under the balanced policy (when it fits the kernel's
  // tables), and under the makespan policy when its simulated time beats the best uniform one.
  if (splits_override == 0 && (policy == PA_POLICY_BALANCED || policy == PA_POLICY_MAKESPAN)) {
    pa::Schedule sch;
    if (pa::build_balanced(*plan, &sch) &&
        (policy == PA_POLICY_BALANCED || sch.makespan_us < plan->est_us * 0.99)) {
      plan->policy = PA_POLICY_BALANCED;
      plan->splits = sch.max_parts;
      plan->units = (int64_t)sch.items.size();
      plan->est_us = (float)sch.makespan_us;
      plan->ws_bytes = (uint64_t)sch.n_slots * sch.rows_per_block * (head_dim + 1) * 4ull;
    }
  }
  return PA_OK;
}

static int write_items(const pa::Schedule& sch, int32_t* items, int cap) {
  const int n = (int)sch.items.size();
  for (int i = 0; i < n && i < cap && items; ++i) {
    items[4 * i + 0] = sch.items[i].rb;
    items[4 * i + 1] = sch.items[i].kt0;
    items[4 * i + 2] = sch.items[i].kt1;
    items[4 * i + 3] = sch.items[i].slot;
  }
  return n;
}

extern "C" int pa_batch_schedule_items(const pa_plan_t* plan, const int32_t* q_lens,
                                       const int64_t* hist_lens, int32_t* items, int cap) {
  if (!plan || plan->batch <= 0 || plan->policy != PA_POLICY_BALANCED) return PA_ERR_INVALID_ARG;
  pa::Batch bt;
  const int st = pa::describe_batch(plan->batch, q_lens, hist_lens, plan->group,
                                    plan->n_kv_heads, plan->ctas_per_unit, &bt);
  if (st != PA_OK) return st;
  pa::Schedule sch;
  if (!pa::build_batch(plan->num_sms, plan->head_dim, plan->ctas_per_unit, plan->group,
                       plan->n_kv_heads, bt, &sch) ||
      (int64_t)sch.items.size() != plan->units)
    return PA_ERR_INVALID_ARG;
  return write_items(sch, items, cap);
}

extern "C" int pa_schedule_items(const pa_plan_t* plan, int32_t* items, int cap) {
  if (!plan || plan->policy != PA_POLICY_BALANCED) return 0;
  if (plan->batch != 0) return PA_ERR_INVALID_ARG;  // pa_batch_schedule_items
  pa::Schedule sch;
  if (!pa::build_balanced(*plan, &sch) || (int64_t)sch.items.size() != plan->units)
    return PA_ERR_INVALID_ARG;
  return write_items(sch, items, cap);
}

extern "C" const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA call failed";
    case PA_ERR_TIMEOUT: return "a kernel wait timed out";
    case PA_ERR_PAGE_INDEX: return "page-table entry out of range";
    default: return "unknown status";
  }
}
