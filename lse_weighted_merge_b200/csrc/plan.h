// plan.h -- host-side argument validation and launch geometry of the merge.
// Pure C++ (no CUDA header), so the planner can be checked on a machine
// without a GPU through lse_merge_plan_query.
#pragma once

#include "lse_merge.h"

namespace lsem {

// Threads per CTA of the throughput (vector) and scalar kernels.
constexpr int kBlock = 256;
// Largest launch the latency path runs as a single CTA (the kernels are
// compiled with __launch_bounds__(kBlock), so one CTA holds at most kBlock).
constexpr int kLatencyMaxThreads = kBlock;

int elem_bytes(int dtype);

// Validate the arguments and fill *plan for `path` (LSE_MERGE_PATH_*).
// Returns LSE_MERGE_OK or the error code lse_merge would return.
int make_plan(const void* partial_o, const float* partial_lse, int R, int B, int H, int D,
              const lse_merge_strides& st, int in_dtype, int out_dtype, const void* out_o,
              const float* out_lse, int path, lse_merge_plan* plan);

// Dense [B,H,R,D] / [B,H,R] strides, used when the caller passes NULL.
lse_merge_strides default_strides(int R, int B, int H, int D);

}  // namespace lsem
