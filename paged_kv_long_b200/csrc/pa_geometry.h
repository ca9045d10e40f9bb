// pa_geometry.h — the work decomposition shared by the planner (host) and the kernels
// (device): packed GQA Q tiles, the keys each tile sees, and the split of those keys.
//
// Source of the decomposition: splash PR #33 ("What changed"): a piece is cut into Q tiles,
// tiles x KV heads x splits are the dispatched units, and the splits partition the history.
// The packing of (token, head) rows is a B200 choice: one 128-row tensor-core tile holds the
// G query heads that share a KV head, so each K/V tile is read once for all of them.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define PA_HD __host__ __device__ __forceinline__
#else
#define PA_HD inline
#endif

namespace pa {

constexpr int kTileRows = 128;   // packed (token, head) rows per Q tile = tensor-core M
constexpr int kTileKeys = 128;   // keys per KV tile = tensor-core N of QK^T, K of PV
constexpr int kMaxSplits = 32;

PA_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Q tiles per KV head for R rows and G heads per KV head.
PA_HD int64_t q_tiles_for(int64_t R, int G) { return ceil_div64(R * G, kTileRows); }

// Decode steps whose group fits one 8-row swizzle atom at head dim 128 or 256 run the kernel
// with swapped operands, two CTAs per SM (pa_decode_plan sizes its splits for those slots).
constexpr int kDecCtasPerSm = 2;
PA_HD bool decode_swapped(int D, int G) { return G <= 8 && (D == 128 || D == 256); }

// Last token (chunk-relative, inclusive) held by Q tile qt.
PA_HD int64_t tile_last_token(int64_t qt, int64_t R, int G) {
  const int64_t t = (qt * kTileRows + kTileRows - 1) / G;
  return t < R - 1 ? t : R - 1;
}

// First token held by Q tile qt.
PA_HD int64_t tile_first_token(int64_t qt, int G) { return (qt * kTileRows) / G; }

// KV tiles visible to Q tile qt: keys [0, H + t_last + 1).
PA_HD int64_t tile_kv_tiles(int64_t qt, int64_t R, int G, int64_t H) {
  return ceil_div64(H + tile_last_token(qt, R, G) + 1, kTileKeys);
}

// KV tiles [*kt0, *kt1) of split s (of S) of a tile that sees n_kt KV tiles.
PA_HD void split_range(int64_t n_kt, int s, int S, int64_t* kt0, int64_t* kt1) {
  *kt0 = (int64_t)s * n_kt / S;
  *kt1 = (int64_t)(s + 1) * n_kt / S;
}

// KV tiles visible to unit-tile qu, when a unit covers `per_unit` consecutive Q tiles (1 or
// 2): those of its last Q tile.
PA_HD int64_t unit_kv_tiles(int64_t qu, int per_unit, int64_t q_tiles, int64_t R, int G,
                            int64_t H) {
  int64_t last = qu * per_unit + per_unit - 1;
  if (last > q_tiles - 1) last = q_tiles - 1;
  return tile_kv_tiles(last, R, G, H);
}

// Unit u -> (Q tile, KV head, split). Units run longest first: the last Q tile (most keys)
// gets the lowest unit indices.
PA_HD void unit_coords(int64_t u, int64_t q_tiles, int Hkv, int S, int64_t* qt, int* g, int* s) {
  const int64_t per_tile = (int64_t)Hkv * S;
  *qt = q_tiles - 1 - u / per_tile;
  const int64_t rem = u % per_tile;
  *g = (int)(rem / S);
  *s = (int)(rem % S);
}

// ---- balanced schedule (plans made with the balanced policy)
//
// A row block is (unit of `per` consecutive Q tiles, KV head): rb = (q_units-1-qu)*Hkv + g,
// longest first. A work item is a contiguous run [kt0, kt1) of a row block's visible KV
// tiles; `slot` is the workspace slot of its partial, or -1 when the item is the whole row
// block and writes the final output.
struct PaItem {
  int32_t rb, kt0, kt1, slot;
};
// Row block that was cut into nparts items, whose partials sit in workspace slots
// [first_slot, first_slot + nparts).
struct PaSplitBlock {
  int32_t rb, first_slot, nparts, pad;
};
constexpr int kMaxItems = 512;
constexpr int kMaxSplitBlocks = 256;

// ---- batched plans (several sequences, each a chunk of `rows` query rows at its own history)
//
// Sequence b owns query/output rows [q_row0, q_row0 + rows) of the packed [sum rows][Hq][D]
// arrays, has `hist` keys before its chunk, and its row blocks are the global row blocks
// [rb0, rb0 + its row-block count), numbered within the sequence as above (longest first).
struct PaSeq {
  int32_t q_row0, rows, hist, rb0;
};
// Batches run on the swapped decode kernel too when every sequence has at most one query row (a
// decode step with host-side lengths) and their row blocks are single CTAs.
inline bool batch_decode_swapped(int D, int G, int per, const PaSeq* seq, int n) {
  if (per != 1 || !decode_swapped(D, G)) return false;
  for (int b = 0; b < n; ++b)
    if (seq[b].rows > 1) return false;
  return true;
}

constexpr int kMaxSeqs = 256;

// The sequence that owns global row block rb: the last b with seq[b].rb0 <= rb (rb0 ascending).
PA_HD int seq_of_rb(const PaSeq* seq, int n, int32_t rb) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq[mid].rb0 <= rb) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

PA_HD void rb_coords(int32_t rb, int64_t q_units, int Hkv, int64_t* qu, int* g) {
  *qu = q_units - 1 - rb / Hkv;
  *g = rb % Hkv;
}

}  // namespace pa
