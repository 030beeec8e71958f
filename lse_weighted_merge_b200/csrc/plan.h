// plan.h -- host-side argument validation and launch geometry of the merge.
// Pure C++ (no CUDA header), so the planner can be checked on a machine
// without a GPU through lse_merge_plan_query.
#pragma once

#include "lse_merge.h"

namespace lsem {

// Threads per CTA of the throughput (vector) and scalar kernels.  Small CTAs
// retire warp by warp: a finished 2-warp CTA frees its registers at once,
// where an 8-warp CTA holds them until its slowest warp ends (measured on
// B200: 64 threads 0.79, 128 threads 0.75, 256 threads 0.71 of the HBM copy
// peak on the R=16 B=512 H=16 D=512 merge, before launch overlap).
#ifndef LSEM_BLOCK
#define LSEM_BLOCK 64
#endif
constexpr int kBlock = LSEM_BLOCK;
// Lower bound on resident CTAs per SM given to __launch_bounds__ (caps registers).
#ifndef LSEM_MINB
#define LSEM_MINB 1
#endif
constexpr int kMinBlocks = LSEM_MINB;
#ifndef LSEM_MINB_VEC1
#define LSEM_MINB_VEC1 LSEM_MINB
#endif
#ifndef LSEM_MINB_STREAM
#define LSEM_MINB_STREAM 0
#endif
constexpr int kMinBlocksVec1 = LSEM_MINB_VEC1;
constexpr int kMinBlocksStream = LSEM_MINB_STREAM;
// Resident CTAs per SM the persistent kernel is compiled for (caps its
// registers; 0 in LSEM_MINB_STREAM picks per instantiation).  Measured on B200
// back to back: the 16-partial kernel (R=16 B=512 H=16 D=512, bf16 -> fp32) at
// 120 registers (8 CTAs of 2 warps per SM) 26.3 us, capped for 8 CTAs (112
// registers, 9 fit) 25.2 us; the 8-partial two-column kernel (rank-major R=8
// B=256 H=64 D=128, fp16) at 158 registers (6 CTAs) 8.9 us, capped for 7 CTAs
// (122 registers, 8 fit) 7.3 us, capped for 8 (128 registers) 7.9 us.
constexpr int stream_min_blocks(int rc, int nv) {
    return kMinBlocksStream > 0 ? kMinBlocksStream : (rc == 8 && nv == 2 ? 7 : 8);
}
// Launch with programmatic stream serialization (the next kernel in the
// stream may be scheduled while this one drains; it waits before touching
// memory).  Hides the launch gap between back-to-back merges.
#ifndef LSEM_PDL
#define LSEM_PDL 1
#endif
constexpr int kPdl = LSEM_PDL;
// Before pdl_wait(), prefetch into L2 the lines of the loads a thread issues
// first, so that a grid launched behind another one starts its first DRAM
// round while the previous grid drains instead of after it has finished.
// 0: off; n > 0: the persistent kernel prefetches its first n row slices,
// the one-shot kernels their first batch of partial rows.
#ifndef LSEM_PREFETCH
#define LSEM_PREFETCH 1
#endif
constexpr int kPrefetch = LSEM_PREFETCH;
// AUTO picks the persistent STREAM kernel from kStreamMinBytes of partials
// (up to kStreamMaxBytes) and the one-shot VECTOR kernel below.  Measured on
// B200: VECTOR is faster below one wave of work (2.1 MB: 2.13 vs 2.36 us
// graph-replayed); with the register caps and the L2 prefetch STREAM is
// faster at every larger size, 606 MB of [B,H,R,D] partials included (96.5
// vs 104.0 us) and 537 MB rank-major (97.3 vs 113.3 us).
#ifndef LSEM_AUTO_STREAM
#define LSEM_AUTO_STREAM 1
#endif
constexpr int kAutoStream = LSEM_AUTO_STREAM;
// AUTO takes R > 16 partials over more than kWideMaxSlices row slices with
// the long form of the persistent kernel (chunks of 16) instead of WIDE.
#ifndef LSEM_AUTO_STREAM_LONG
#define LSEM_AUTO_STREAM_LONG 1
#endif
constexpr int kAutoStreamLong = LSEM_AUTO_STREAM_LONG;
// Threads (one 16-byte column per lane) from which AUTO prefers the long form
// for R > 16: about 0.6 of a B200 wave (148 SMs x 8 CTAs x 64 threads).
// Measured, graph-replayed: R=24 over 4096 rows of D=128 (65536 threads) long
// 7.7 us, WIDE 8.6; R=32 over 2048 rows (32768) long 6.3, WIDE 5.3; R=64 over
// 2048 rows 10.3 and 10.2; R=128 over 512 rows long 13.5, WIDE 5.6.
constexpr long long kLongMinThreads = 48 * 1024;
#ifndef LSEM_STREAM_MAX_MB
#define LSEM_STREAM_MAX_MB (1 << 30)
#endif
constexpr long long kStreamMaxBytes = (long long)LSEM_STREAM_MAX_MB << 20;
constexpr long long kStreamMinBytes = 8ll << 20;
// Row slices up to which AUTO spreads each row over a CTA (WIDE) even for
// R <= 16: a handful of rows is latency-bound, and more threads per row beat
// more loads per thread (8 rows of R=8: 2.03 us WIDE, 2.23 us VECTOR).
constexpr long long kWideMaxSlices = 128;
// Most threads per CTA of the wide kernel (one CTA per row slice).
constexpr int kWideBlock = 128;
// Upper bound on the 16-byte columns per lane (1, 2 or 4).
#ifndef LSEM_MAX_NV
#define LSEM_MAX_NV 2
#endif
constexpr int kMaxNv = LSEM_MAX_NV;
// When the last round of a full persistent grid would be less than half
// full, size the grid so that every CTA gets the same number of rounds
// (ceil(work / capacity) rounds, spread evenly); see balanced() in
// lse_merge.cu.  0 always fills the device.
#ifndef LSEM_BALANCE
#define LSEM_BALANCE 1
#endif
constexpr int kBalance = LSEM_BALANCE;
// Largest launch the latency path runs as a single CTA (the kernels are
// compiled with __launch_bounds__(kBlock), so one CTA holds at most kBlock).
constexpr int kLatencyMaxThreads = kBlock;

int elem_bytes(int dtype);

// The cudaError_t of the last failed launch on this host thread.
void set_last_cuda_error(int e);
int last_cuda_error();

// Validate the arguments and fill *plan for `path` (LSE_MERGE_PATH_*).
// Returns LSE_MERGE_OK or the error code lse_merge would return.
int make_plan(const void* partial_o, const float* partial_lse, int R, int B, int H, int D,
              const lse_merge_strides& st, int in_dtype, int out_dtype, const void* out_o,
              const float* out_lse, int path, lse_merge_plan* plan);

// Dense [B,H,R,D] / [B,H,R] strides, used when the caller passes NULL.
lse_merge_strides default_strides(int R, int B, int H, int D);

// Launch geometry of the in-place state update: a group of `lanes` lanes per
// row, lane j folding the 8-element chunks j, j + lanes, ... of the row.
struct StatePlan {
    int vec;        // 1: 16-byte loads and stores; 0: element accesses
    int lanes;      // power of two <= 32
    int chunks;     // 8-element chunks per row, ceil(D / 8)
    int block;
    int64_t grid;
};

// Decode attention: what the kernel does with each split's partial.
constexpr int kAttnModePartials = 0;    // writes it to the caller's partial buffers
constexpr int kAttnModeCluster = 1;     // hands it to CTA 0 of the cluster, which merges
constexpr int kAttnModeWorkspace = 2;   // workspace + counter: the last split merges

// Decode attention: validated geometry.
struct AttnPlan {
    int G;            // query heads per KV head
    int mode;         // kAttnMode*
    int64_t smem;     // dynamic shared memory per CTA
    // workspace (kAttnModeWorkspace): counters [B, Hkv] u32 at 0, split lse
    // [B, Hkv, R, G] f32 at ws_l_off, split o [B, Hkv, R, G, D] f32 at ws_o_off
    int64_t ws_l_off, ws_o_off, ws_bytes;
};
constexpr int kAttnWarps = 4;     // warps per CTA, each a private K/V ring
#ifndef LSEM_ATTN_TK
#define LSEM_ATTN_TK 16
#endif
#ifndef LSEM_ATTN_STAGES
#define LSEM_ATTN_STAGES 3
#endif
constexpr int kAttnTileKeys = LSEM_ATTN_TK;    // keys per K/V tile (16 or 32)
constexpr int64_t kAttnMaxSmem = 227 * 1024;   // dynamic shared memory one CTA may take
constexpr int kAttnStages = LSEM_ATTN_STAGES;  // tiles per warp ring

int make_attn_plan(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int L,
                   int D, int R, float scale, const lse_merge_attn_strides& st, int dtype,
                   int out_dtype, const void* out_o, const float* out_lse, int mode,
                   const void* ws, int64_t ws_bytes, AttnPlan* plan);
// Workspace layout of kAttnModeWorkspace for these sizes (no pointer checks).
int attn_workspace_layout(int B, int Hq, int Hkv, int R, int D, AttnPlan* plan);
lse_merge_attn_strides default_attn_strides(int Hq, int Hkv, int L, int D);

// Validate the arguments of lse_merge_state_update and fill *plan.
int make_state_plan(const void* o_acc, const float* lse_acc, const void* o_new,
                    const float* lse_new, int B, int H, int D, const lse_merge_state_strides& st,
                    int acc_dtype, int new_dtype, StatePlan* plan);

// Context-parallel exchange + merge: validated layout of one rank's workspace
// and of the units each rank sends.  A unit is 16 bytes of one partial row.
struct CpPlan {
    int world, rank_begin, rank_count, Hq;
    int in_bytes, out_bytes;
    int dv;            // units per row, D * in_bytes / 16
    int64_t U;         // units one rank sends to one other rank, B * Hq * dv
    int64_t slot_o;    // bytes of one received partial block [B, Hq, D]
    int64_t slot_l;    // bytes of one received lse block [B, Hq]
    int64_t o_off;     // workspace offset of recv_o [2][world-1][B][Hq][D]
    int64_t l_off;     // workspace offset of recv_lse [2][world-1][B][Hq]
    int64_t ws_bytes;  // bytes of one workspace
};
constexpr int kCpBlock = 256;
constexpr int64_t kCpHeaderBytes = 256;   // counters and status word of a workspace
constexpr int64_t kCpMaxTimeoutNs = 60ll * 1000 * 1000 * 1000;

// Workspace layout for these sizes (no pointer checks).
int cp_layout(int world, int B, int H, int D, int in_dtype, CpPlan* plan);
// Full validation of lse_merge_cp_exchange_merge's arguments.
int make_cp_plan(const lse_merge_cp_args& a, CpPlan* plan);

}  // namespace lsem
