// Host-side launch plan of spa_attention.
#pragma once

#include <stddef.h>

#include "spa.h"

namespace spa {

enum PlanKind { kPlanScalar = 0, kPlanMma = 1, kPlanPrefill = 2, kPlanTc = 3 };

struct Plan {
  int kind;
  int group_by_request;
  int max_q;
  int max_rows;
  int num_splits;
  int split_len;
  int units;
  int cluster_merge;  // splits of a unit merge after a cluster barrier (no tickets)
  size_t ws_acc_bytes;
  size_t ws_ml_bytes;
  size_t ws_count_bytes;
};

int validate_attention(const spa_attention_args_t* a);
int make_plan(const spa_attention_args_t* a, Plan* pl);

}  // namespace spa
