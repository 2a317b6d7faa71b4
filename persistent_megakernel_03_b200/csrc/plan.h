// plan.h -- host-side task-graph (tGraph) builder.
#pragma once
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

namespace mk {

struct Plan {
  int num_ctas = 0;
  int attn_splits = 1;
  int n_lm_tasks = 0;
  int n_lm_slots = 0;                      // CTAs holding LM-head tasks
  int n_events = 0;
  int n_tickets = 0;
  int n_stages = 0;
  int lm_ticket = 0;
  std::vector<Task> tasks;                 // w == nullptr until the context patches it
  std::vector<int> cta_of_task;
  std::vector<uint32_t> event_count;       // signals per step
  // queue sets: set 0 = megakernel (all tasks), set 1 + s = stage s only
  std::vector<int> queue;                  // task indices
  std::vector<int> queue_off;              // [(n_stages + 1) * (num_ctas + 1)]
  long long weight_bytes = 0;

  int set_offset(int set) const { return set * (num_ctas + 1); }
};

// Validates cfg; on error returns a message.
std::string validate_config(const mk_config& c);

// Builds the task graph for `num_ctas` CTAs.  attn_splits <= 0: automatic.
// wbytes: bytes per GEMV weight (2 bf16, 1 fp8); a task's geometry (threads
// per row, rows per ring chunk, rows per task) follows the bytes of a row.
std::string build_plan(const mk_config& c, int num_ctas, int attn_splits, Plan* out, int wbytes = 2);

// Event indices.
struct EventMap {
  int L, nkv;
  int qkv(int l, int g) const { return l * nkv + g; }
  int attn(int l) const { return L * nkv + l; }
  int oproj(int l) const { return L * nkv + L + l; }
  int gateup(int l) const { return L * nkv + 2 * L + l; }
  int down(int l) const { return L * nkv + 3 * L + l; }
  int count() const { return L * nkv + 4 * L; }
};

}  // namespace mk
