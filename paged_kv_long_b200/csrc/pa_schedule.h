// pa_schedule.h — host side of the balanced schedule: the item list of a plan made with the
// balanced policy, rebuilt deterministically from the plan's fields by the planner, the prefill
// launch and the combine launch.
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

}  // namespace pa
