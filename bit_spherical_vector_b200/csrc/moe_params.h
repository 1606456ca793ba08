// moe_params.h -- parameter block and workspace layout of the grouped MoE GEMV.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "svq.h"

namespace svq {

struct MoeKParams {
  const svq_matrix* mats;          // device array [n_mats], all N x K
  int n_mats, N, K, max_b_d;
  const svq_group_item* items;     // device array [n_items]
  int n_items;
  const void* x;                   // x_mode 0: fp16 [*][K]; 1: fp32 [*][2K] (gate | up)
  int x_mode;
  int n_x_rows;                    // rows of x (items' x_row must be below)
  float* y;                        // [n_out_rows][N]
  int n_out_rows;
  int accumulate;
  int* offsets;                    // workspace: item offsets per matrix [n_mats + 1]
  int* cursor;                     // [n_mats]
  int* sorted;                     // item indices grouped by matrix [n_items]
  int* active;                     // touched matrices [n_mats]
  int* n_active;                   // [1]
  int* costpre;                    // [n_mats + 1]: cost prefix over the active list (balances CTAs)
  int mt;                          // items per decode pass of the kernel (1, 2 or 4)
  int local_route;                 // 1: every CTA builds the routing tables in shared memory
  float* item_out;                 // [n_items][N] (accumulate only)
  int* status;                     // device status word
};

struct MoeWorkspace {
  size_t offsets, cursor, sorted, active, n_active, costpre, item_out, total;
};

MoeWorkspace moe_workspace_layout(int n_mats, int n_items, int N, int accumulate);
// Whether the routing tables are small enough to be built by every CTA in
// shared memory (no separate routing kernel).
bool moe_local_route(int n_mats, int n_items);
size_t moe_smem_bytes(int max_b_d, int K, int mt, int n_mats, int n_items);
cudaError_t launch_moe(MoeKParams p, int mt, int n_out_rows, int num_sms, cudaStream_t st);

}  // namespace svq
