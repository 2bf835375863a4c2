// Internal declarations of the device-side EAGLE-2 draft tree (tsd_draft_tree_*).
#pragma once

#include "kernels.h"

namespace tsd {

struct DraftTreeArgs {
  int32_t* parent;        // [B, max_nodes]
  int32_t* token;         // [B, max_nodes]
  double* score;          // [B, max_nodes] cumulative draft log-probability
  int32_t* depth;         // [B, max_nodes]
  int32_t* num_nodes;     // [B]
  int32_t* frontier;      // [B, F] node ids, best first
  int32_t* num_frontier;  // [B]
  int max_nodes, F, B;
};
size_t draft_expand_ws(int B, int F, int K, int V);
tsd_status launch_draft_init(const DraftTreeArgs& t, const int32_t* root_token, int32_t* status, cudaStream_t stream);
tsd_status launch_draft_expand(const DraftTreeArgs& t, const void* logits, tsd_dtype dtype, int V, int K, void* ws,
                               int32_t* status, cudaStream_t stream);
tsd_status launch_draft_finalize(const DraftTreeArgs& t, int keep, int32_t* parent_out, int32_t* tokens_out,
                                 int32_t* num_out, int32_t* status, cudaStream_t stream);

}  // namespace tsd
