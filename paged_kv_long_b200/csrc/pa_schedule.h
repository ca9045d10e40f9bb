// pa_schedule.h — host side of the balanced schedule: the item list of a plan made with the
// balanced policy, rebuilt deterministically from the plan's fields (and, for a batch, the
// sequences' lengths) by the planner, the prefill launch and the combine launch.
#pragma once
#include <vector>

#include "pa.h"
#include "pa_geometry.h"

namespace pa {

struct Schedule {
  std::vector<PaItem> items;          // in launch order
  std::vector<PaSplitBlock> split;    // row blocks with more than one item
  int32_t n_slots = 0;                // workspace slots (partials)
  int32_t rows_per_block = 0;         // packed rows of a row block (per * 128)
  int32_t max_parts = 1;
  double makespan_us = 0.0;           // simulated
};

// Fills `out` for the piece described by `p` (its shape fields; the policy is not read).
// Returns false when the schedule would exceed the kernel's item or split-block tables.
bool build_balanced(const pa_plan_t& p, Schedule* out);

// A batch of sequences: sequence b has q_lens[b] query rows after hist_lens[b] keys.
struct Batch {
  std::vector<PaSeq> seq;   // q_row0, rows, hist, rb0 of every sequence
  int64_t total_rows = 0;   // sum of q_lens
  int64_t row_blocks = 0;   // sum of the sequences' row blocks
  int64_t max_hist = 0;
};
// Validates the lengths and lays the sequences out (rows packed in order). Returns a pa_status.
int describe_batch(int batch, const int32_t* q_lens, const int64_t* hist_lens, int G, int Hkv,
                   int per, Batch* out);
// CTAs per row block of a batch: 2 (CTA pairs, head dim 256) only when some sequence has two
// or more Q tiles; a batch of one-tile sequences (decode) would leave half of every pair idle.
int batch_ctas_per_unit(int head_dim, int G, int batch, const int32_t* q_lens);
// The balanced schedule of a batch (row blocks of all sequences, longest first).
bool build_batch(int num_sms, int head_dim, int per, int G, int Hkv, const Batch& bt,
                 Schedule* out);

}  // namespace pa
