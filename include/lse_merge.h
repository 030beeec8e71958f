/*
 * lse_merge.h -- C ABI of the B200 (sm_100a) LSE-weighted merge.
 *
 * The operation.  Under context-parallel decode the KV cache is split along
 * the sequence into R shards; attention over shard r yields a partial output
 * o_r[D] and lse_r, the natural-log log-sum-exp of that shard's scores (page
 * "[flashinfer] FlashInfer의 Context-Parallel Decode 최적화: Fused A2A + LSE
 * Reduce", section "들어가며").  The merge combines the R partials of every
 * (b, h) row into the output of attention over the whole sequence: weights
 * from the lse values, fp32 accumulation over the partial axis, division by
 * the sum of the weights, conversion to the output type (same page, section
 * "코드 분석 / 1. Fused Kernel 구현", its Before/After snippet and the fused
 * kernel's steps 2 and 3).  Per row:
 *
 *     m       = max_r lse_r
 *     e_r     = exp(lse_r - m)          (0 when lse_r = -inf: an empty shard)
 *     out[d]  = sum_r e_r * o_r[d] / sum_r e_r
 *     out_lse = m + log(sum_r e_r)
 *
 * and out = 0, out_lse = -inf for a row whose shards are all empty.  The
 * partial rows of an empty shard do not reach the result (NaN there does not
 * leak).  lse = +inf or NaN is outside the domain; NaN then propagates.
 *
 * Everything runs on the GPU inside one kernel launch per call; the library
 * allocates nothing, keeps no pointer after returning, never synchronises
 * the host, and only enqueues work on `stream`, so a call can be captured in
 * a CUDA graph.  The exceptions are the set-up calls of the context-parallel
 * exchange (lse_merge_cp_workspace_create and the IPC calls) and of the
 * host-buffer merge (lse_merge_host_create / _destroy), which say so.
 */
#ifndef LSE_MERGE_H
#define LSE_MERGE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of partial_o and out_o.  lse values are always fp32. */
typedef enum {
    LSE_MERGE_F32 = 0,
    LSE_MERGE_F16 = 1,   /* IEEE binary16 */
    LSE_MERGE_BF16 = 2   /* bfloat16 */
} lse_merge_dtype;

/* The same type as cudaStream_t; declared here so that this header needs no
 * CUDA header.  NULL is the legacy default stream. */
typedef struct CUstream_st* lse_merge_stream_t;

/* Element (not byte) strides of the two inputs along r, b and h.  The d
 * stride of partial_o is 1.  All strides must be >= 0.  Examples with dense
 * storage:
 *   partial_o [B,H,R,D], partial_lse [B,H,R]:  o = {D, H*R*D, R*D},  lse = {1, H*R, R}
 *   partial_o [R,B,H,D], partial_lse [R,B,H]:  o = {B*H*D, H*D, D},  lse = {B*H, H, 1}  */
typedef struct {
    int64_t o_r, o_b, o_h;
    int64_t lse_r, lse_b, lse_h;
} lse_merge_strides;

/* Return codes.  No error is ever reported by a device trap or by an
 * exception crossing the ABI. */
#define LSE_MERGE_OK 0
#define LSE_MERGE_EDTYPE (-1)   /* in_dtype / out_dtype not one of lse_merge_dtype */
#define LSE_MERGE_EDIMS (-2)    /* R, B, H or D < 1, or the extents overflow */
#define LSE_MERGE_ENULL (-3)    /* a required pointer is NULL */
#define LSE_MERGE_ESTRIDE (-4)  /* a negative stride */
#define LSE_MERGE_EALIAS (-5)   /* an output overlaps an input or the other output */
#define LSE_MERGE_ELAUNCH (-6)  /* the CUDA launch failed (see lse_merge_last_cuda_error) */
#define LSE_MERGE_EALIGN (-7)   /* a pointer not aligned to its element size */
#define LSE_MERGE_EPATH (-8)    /* the requested path cannot take these arguments */
#define LSE_MERGE_EUNSUP (-9)   /* a shape the decode-attention kernels do not implement */
#define LSE_MERGE_ECUDA (-10)   /* a CUDA runtime call of a set-up function failed */
#define LSE_MERGE_ESCRATCH (-11) /* the problem needs more than the static scratch holds */
#define LSE_MERGE_EDEVICE (-12)  /* the current device is not the one the context was made on */

/* Kernel paths.  AUTO picks one from the sizes, dtypes and alignment. */
#define LSE_MERGE_PATH_AUTO 0
#define LSE_MERGE_PATH_VECTOR 1   /* 16-byte vector loads, many CTAs (throughput) */
#define LSE_MERGE_PATH_LATENCY 2  /* the vector kernel as one small CTA (tiny B*H) */
#define LSE_MERGE_PATH_SCALAR 3   /* element loads, any alignment of strides and D */
#define LSE_MERGE_PATH_STREAM 4   /* persistent vector kernel, loads of the next row slice
                                     issued as the current one is consumed; R > 16 in
                                     chunks of partials with a running max */
#define LSE_MERGE_PATH_WIDE 5     /* one CTA per row slice, the partials spread over its
                                     lane groups and their states merged (large R, few rows) */

/*
 * Merge R partials of B*H rows.
 *
 *   partial_o    device pointer, element (r,b,h,d) at
 *                r*o_r + b*o_b + h*o_h + d (elements of in_dtype)
 *   partial_lse  device pointer, element (r,b,h) at r*lse_r + b*lse_b + h*lse_h
 *   R, B, H, D   partials per row, batch, heads, head dimension; all >= 1
 *   strides      as above; NULL means dense [B,H,R,D] / [B,H,R]
 *   in_dtype     element type of partial_o (lse_merge_dtype)
 *   out_dtype    element type of out_o (lse_merge_dtype)
 *   out_o        device pointer, dense [B,H,D] of out_dtype, written
 *   out_lse      device pointer, dense [B,H] fp32, written
 *   stream       CUDA stream the kernel is enqueued on; it and every pointer
 *                belong to the calling thread's current CUDA device
 *
 * The caller owns every buffer.  Pointers must be aligned to their element
 * size; the fast path additionally wants 16-byte aligned partial_o rows and
 * falls back to the scalar kernel otherwise.  Outputs must not overlap the
 * inputs or each other.  Returns LSE_MERGE_OK, or a negative code with
 * nothing enqueued (argument errors) or after a failed launch (ELAUNCH).
 */
int lse_merge(const void* partial_o, const float* partial_lse,
              int R, int B, int H, int D,
              const lse_merge_strides* strides,
              int in_dtype, int out_dtype,
              void* out_o, float* out_lse,
              lse_merge_stream_t stream);

/* lse_merge with an explicit kernel path (one of LSE_MERGE_PATH_*).  Returns
 * LSE_MERGE_EPATH when that path cannot take the arguments (for example the
 * vector path with a misaligned stride).  Meant for tests and benchmarks. */
int lse_merge_with_path(const void* partial_o, const float* partial_lse,
                        int R, int B, int H, int D,
                        const lse_merge_strides* strides,
                        int in_dtype, int out_dtype,
                        void* out_o, float* out_lse,
                        lse_merge_stream_t stream, int path);

/* The launch plan lse_merge_with_path would use.  Host-only: validates the
 * arguments exactly as lse_merge does (pointers are only inspected, never
 * dereferenced) and fills *plan without touching the GPU. */
typedef struct {
    int path;            /* LSE_MERGE_PATH_VECTOR / _LATENCY / _SCALAR / _STREAM / _WIDE */
    int vec;             /* elements per lane per partial load (16 B / elem size; 1 for scalar) */
    int lanes;           /* lanes that share one row slice (power of two, <= 32) */
    int rc;              /* partial rows whose loads are in flight together per lane */
    int nv;              /* 16-byte columns per lane in every partial row (rc * nv <= 16) */
    int slices_per_row;  /* row slices (lane groups) that cover one row of D */
    int block;           /* threads per CTA */
    int64_t grid;        /* CTAs; 0 for STREAM, whose persistent grid is sized at
                            launch to the CTAs that fit on the device at once */
    int64_t groups;      /* row slices in total: B*H*slices_per_row */
} lse_merge_plan;

int lse_merge_plan_query(const void* partial_o, const float* partial_lse,
                         int R, int B, int H, int D,
                         const lse_merge_strides* strides,
                         int in_dtype, int out_dtype,
                         const void* out_o, const float* out_lse,
                         int path, lse_merge_plan* plan);

/*
 * Fold one new partial into an accumulator, in place (the merge above with
 * R = 2 whose first partial is the accumulator; applied shard after shard it
 * gives the R-way merge, because the log-sum-exp combine is associative).
 * Per row (b, h):
 *
 *     m       = max(lse_acc, lse_new)
 *     e_a     = exp(lse_acc - m),  e_n = exp(lse_new - m)    (0 for -inf)
 *     o_acc   = (e_a * o_acc + e_n * o_new) / (e_a + e_n)
 *     lse_acc = m + log(e_a + e_n)
 *
 * and 0, -inf when both sides are empty.  The values of an empty side never
 * reach the result (NaN there does not leak), so an accumulator can start as
 * lse_acc = -inf with o_acc uninitialised.  The pages
 * describe the R-way merge only; this entry point is derived from it.
 *
 *   o_acc, lse_acc  device pointers, dense [B,H,D] of acc_dtype and [B,H] fp32;
 *                   read and overwritten
 *   o_new, lse_new  device pointers; element (b,h,d) of o_new at
 *                   b*o_b + h*o_h + d, element (b,h) of lse_new at
 *                   b*lse_b + h*lse_h (new_strides; NULL = dense [B,H,D], [B,H])
 *   acc_dtype, new_dtype   lse_merge_dtype of o_acc and o_new
 *   stream          as for lse_merge
 *
 * The new partial must not overlap the accumulator, nor o_acc lse_acc.
 * Returns the codes of lse_merge (LSE_MERGE_EPATH does not occur).
 */
typedef struct {
    int64_t o_b, o_h;
    int64_t lse_b, lse_h;
} lse_merge_state_strides;

int lse_merge_state_update(void* o_acc, float* lse_acc, const void* o_new, const float* lse_new,
                           int B, int H, int D, const lse_merge_state_strides* new_strides,
                           int acc_dtype, int new_dtype, lse_merge_stream_t stream);

/*
 * Split-KV decode attention, the producer of the partials (the CP-decode
 * page's introduction: each rank attends over its own KV shard and returns
 * o_r and lse_r).  One query token per sequence, grouped heads: query head h
 * attends over KV head h / (Hq / Hkv).  The keys [0, len_b) of sequence b
 * (len_b = kv_len[b] clamped to [0, L], or L when kv_len is NULL) are cut into
 * R splits of ceil(len_b / R) keys; split r is the shard [r*ceil, min(len_b,
 * (r+1)*ceil)).  For a split with keys j:
 *
 *     s_j = scale * <q, k_j>,  lse_r = log sum_j exp(s_j),
 *     o_r = sum_j exp(s_j - lse_r) * v_j        (empty split: 0 and -inf)
 *
 *   q        [B, Hq, D]: element (b,h,d) at b*q_b + h*q_h + d
 *   k, v     [B, Hkv, L, D]: element (b,h,l,d) at b*k_b + h*k_h + l*k_l + d
 *            (v likewise with v_*); strides in elements, d stride 1; NULL
 *            strides = dense
 *   dtype    LSE_MERGE_BF16 or LSE_MERGE_F16 (q, k and v)
 *   D        64 or 128; Hq a multiple of Hkv with Hq / Hkv <= 16
 *   q, k, v  16-byte aligned, with strides of whole 16-byte multiples
 *
 * lse_merge_decode_partials writes the R partials, fp32, into caller buffers
 * dense [B, Hq, R, D] and [B, Hq, R] (the layout lse_merge takes as its
 * default), for a separate merge.
 *
 * lse_merge_decode_attention also merges them, inside the same kernel: the
 * R CTAs of one (b, KV head) form a thread-block cluster; CTAs 1..R-1 store
 * their split's partial into CTA 0's shared memory (distributed shared
 * memory) and exit, and CTA 0 merges the R partials, so the partials never
 * reach HBM.  R must be 1, 2, 4 or 8.  Output out_o dense [B, Hq, D] of
 * out_dtype and out_lse dense [B, Hq] fp32: attention over keys [0, len_b).
 * CTA 0's wait for the other partials is bounded (2 s); should it ever run
 * out, that row's outputs are NaN instead of the kernel hanging.
 *
 * lse_merge_decode_attention_ws merges them in the same kernel without a
 * cluster, through a caller workspace of lse_merge_decode_workspace_bytes()
 * bytes (16-byte aligned, overlapping no other argument): each split CTA
 * stores its fp32 partial there and counts itself in a per-(b, KV head)
 * counter; the CTA that completes the count merges the R partials (still in
 * L2) and resets the counter.  No CTA waits for another, and any R >= 1 is
 * accepted.  The workspace must be zeroed once before its first use; every
 * call leaves it ready for the next one (counters back at 0).  Calls that
 * may run at the same time on the GPU need workspaces of their own, and a
 * call that did not complete (a launch error) requires zeroing it again.
 * Output as for lse_merge_decode_attention.
 *
 * All return the codes of lse_merge, and LSE_MERGE_EUNSUP for a D, group
 * size, dtype or R outside the above; the workspace form also EDIMS for a
 * workspace shorter than lse_merge_decode_workspace_bytes().
 */
typedef struct {
    int64_t q_b, q_h;
    int64_t k_b, k_h, k_l;
    int64_t v_b, v_h, v_l;
} lse_merge_attn_strides;

int lse_merge_decode_partials(const void* q, const void* k, const void* v, const int32_t* kv_len,
                              int B, int Hq, int Hkv, int L, int D, int R, float scale,
                              const lse_merge_attn_strides* strides, int dtype,
                              float* partial_o, float* partial_lse, lse_merge_stream_t stream);

int lse_merge_decode_attention(const void* q, const void* k, const void* v, const int32_t* kv_len,
                               int B, int Hq, int Hkv, int L, int D, int R, float scale,
                               const lse_merge_attn_strides* strides, int dtype, int out_dtype,
                               void* out_o, float* out_lse, lse_merge_stream_t stream);

/* Bytes of the workspace of lse_merge_decode_attention_ws: counters [B, Hkv]
 * (uint32), then the split lse [B, Hq, R] and o [B, Hq, R, D] (fp32). */
int lse_merge_decode_workspace_bytes(int B, int Hq, int Hkv, int R, int D, int64_t* bytes);

int lse_merge_decode_attention_ws(const void* q, const void* k, const void* v,
                                  const int32_t* kv_len, int B, int Hq, int Hkv, int L, int D,
                                  int R, float scale, const lse_merge_attn_strides* strides,
                                  int dtype, int out_dtype, void* workspace,
                                  int64_t workspace_bytes, void* out_o, float* out_lse,
                                  lse_merge_stream_t stream);

/* ---------------------------------------------------------------------------
 * Context-parallel exchange and merge in one kernel.
 *
 * The step before the merge on the CP-decode page (section "코드 분석 / 1.
 * Fused Kernel 구현": instead of an all-to-all followed by a separate merge,
 * each rank writes its partials straight into the buffer of the rank that
 * owns them, and the owner merges once everything has landed; the
 * introduction, "들어가며", gives the partials themselves).  `world` ranks
 * each hold the partials of their own KV shard for all B*H rows:
 *   local_o [B,H,D] of in_dtype, dense;  local_lse [B,H] fp32, dense.
 * Heads are scattered in equal contiguous blocks: rank q owns heads
 * [q*Hq, (q+1)*Hq) with Hq = H / world, and produces
 *   out_o [B,Hq,D] of out_dtype, dense;  out_lse [B,Hq] fp32, dense,
 * the merge over all ranks' partials of its heads.  One launch, per rank:
 *   1. every (b, h) row owned by another rank q is stored into q's workspace
 *      (plain 16-byte stores; ws[q] may be a peer GPU's memory);
 *   2. the rank adds the number of 16-byte units it stored for q to q's
 *      landed counter for this sender (a system-scope release; device scope
 *      when the launch plays every rank);
 *   3. it waits, bounded by timeout_ns of the GPU's global timer, until every
 *      other rank's landed counter in its own workspace reached e * U, e the
 *      number of this call since the workspace was zeroed (U = B*Hq*D*elem/16
 *      units per sender);
 *   4. it merges its rows: its own partial read in place from local_o, the
 *      others from its workspace;
 *   5. its last CTA to finish records call e as completed in the workspace.
 * The call number lives in the workspace, so every rank must make the same
 * calls since the workspaces were zeroed, each rank's calls ordered on one
 * stream; a captured CUDA graph may replay a call.  Across GPUs, received
 * rows alternate between two slots by the parity of e, so a rank may start
 * call e + 1 while a peer still merges call e; a launch that plays every rank
 * uses one slot, since its next call starts after it ends.  A wait that runs out ORs bit s (sender s) into
 * the uint32 status word at byte LSE_MERGE_CP_STATUS_OFFSET of that rank's
 * workspace, leaves that rank's outputs unwritten and returns; the
 * workspaces are then out of step, and every rank must zero its workspace
 * (lse_merge_cp_workspace_zero) before the next call.
 *
 * One launch may play several ranks: ranks rank_begin .. rank_begin +
 * rank_count - 1 (local_o[i], local_lse[i], out_o[i], out_lse[i] belong to
 * rank rank_begin + i).  All CTAs of a launch are co-resident (cooperative
 * launch), so a single GPU can play all `world` ranks at once; in a multi-GPU
 * job each process plays its own rank (rank_count = 1) and ws[] holds the
 * peers' workspaces (lse_merge_cp_ipc_open).
 *
 * Requirements: 1 <= world <= LSE_MERGE_CP_MAX_WORLD; H % world == 0;
 * D * elem(in_dtype) a multiple of 16 bytes; B*H*D*elem(in_dtype) below
 * 32 GiB (2^31 units of 16 bytes); 0 <= rank_begin and
 * rank_begin + rank_count <= world; local_o and out_o 16-byte aligned, lse
 * pointers 4-byte aligned, workspaces 256-byte aligned and
 * lse_merge_cp_workspace_bytes() long (zeroed before the first call);
 * 0 < timeout_ns <= 60 s.  Outputs may not overlap inputs or workspaces.  The
 * library keeps no pointer.  Returns the codes of lse_merge (EDIMS for the
 * requirements on world, H, the ranks and the timeout, EALIGN for D and the
 * pointers) and LSE_MERGE_ELAUNCH when the launch fails, e.g. a grid that
 * cannot be co-resident.
 */
#define LSE_MERGE_CP_MAX_WORLD 8
#define LSE_MERGE_CP_STATUS_OFFSET 64     /* uint32 in each workspace; 0 = no wait ran out */
#define LSE_MERGE_CP_IPC_HANDLE_BYTES 64
/* Run the cross-GPU protocol (system-scope release and acquire, two receive
 * slots) even when the launch plays every rank, which otherwise uses device
 * scope and one slot; this lets one GPU test the multi-GPU protocol. */
#define LSE_MERGE_CP_FLAG_CROSS_GPU_PROTOCOL 1
/* For tests of the failure path only: the highest-numbered rank of the call
 * sends nothing, so every other rank's bounded wait for it runs out after
 * timeout_ns, sets that sender's bit in the rank's status word and skips
 * the rank's merge.  The kernel still ends on its own; nothing faults. */
#define LSE_MERGE_CP_FLAG_TEST_SILENT_LAST_RANK 2

typedef struct {
    int world, rank_begin, rank_count;
    const void* local_o[LSE_MERGE_CP_MAX_WORLD];    /* per played rank */
    const float* local_lse[LSE_MERGE_CP_MAX_WORLD];
    void* out_o[LSE_MERGE_CP_MAX_WORLD];            /* per played rank */
    float* out_lse[LSE_MERGE_CP_MAX_WORLD];
    void* ws[LSE_MERGE_CP_MAX_WORLD];               /* workspace of every rank q < world */
    int B, H, D, in_dtype, out_dtype;
    int64_t timeout_ns;
    int flags;                                      /* LSE_MERGE_CP_FLAG_*, normally 0 */
} lse_merge_cp_args;

/* Bytes of one rank's workspace (the same on every rank). */
int lse_merge_cp_workspace_bytes(int world, int B, int H, int D, int in_dtype, int64_t* bytes);
/* Check the arguments as lse_merge_cp_exchange_merge does, without a GPU. */
int lse_merge_cp_validate(const lse_merge_cp_args* args);
int lse_merge_cp_exchange_merge(const lse_merge_cp_args* args, lse_merge_stream_t stream);

/* Workspaces shared between processes (one GPU per process).  create:
 * cudaMalloc of `bytes` on the current device, zeroed before it returns.
 * ipc_handle: the cudaIpcMemHandle_t of a created workspace, copied into
 * `handle` (LSE_MERGE_CP_IPC_HANDLE_BYTES bytes).  ipc_open: maps a peer's
 * workspace into this process (peer access enabled), *peer_ws its address;
 * ipc_close unmaps it.  These are set-up calls: they synchronise the device,
 * and create is the one place the library allocates.  They return
 * LSE_MERGE_ECUDA when the CUDA call fails (lse_merge_last_cuda_error). */
int lse_merge_cp_workspace_create(int64_t bytes, void** ws);
/* The status word of a workspace (0 = no wait ran out, bit s = sender s never
 * landed) and the restart after a wait ran out: zero `bytes` of the
 * workspace.  Both first wait for all work on the current device, on every
 * stream, then copy or zero synchronously.  Before zeroing, every rank must
 * also know that no peer's kernel still writes into this workspace (the
 * Python group synchronises every device, then passes a barrier). */
int lse_merge_cp_status(const void* ws, uint32_t* status);
int lse_merge_cp_workspace_zero(void* ws, int64_t bytes);
int lse_merge_cp_workspace_destroy(void* ws);
int lse_merge_cp_ipc_handle(void* ws, void* handle);
int lse_merge_cp_ipc_open(const void* handle, void** peer_ws);
int lse_merge_cp_ipc_close(void* peer_ws);

/* The exchange and merge for callers that cannot allocate device memory.
 * (No counterpart on the pages; it is a service of this library.)
 *
 * Some callers cannot call cudaMalloc at the point where they run this step:
 * a serving runtime that has handed all spare HBM to its KV-cache pool at
 * start-up has nothing left to allocate, and cudaMalloc itself may
 * synchronise the whole device, which a decode step that must keep the
 * device busy cannot afford.  This entry point therefore allocates nothing:
 * the workspaces of all ranks are carved out of one array that the library
 * defines in device memory, LSE_MERGE_CP_NOALLOC_SCRATCH_BYTES (16 MiB) per
 * GPU, held by every GPU that loads the library until the process exits.
 * The caller passes inputs and outputs exactly as for
 * lse_merge_cp_exchange_merge, with these differences:
 *   - the launch must play every rank (rank_begin = 0, rank_count = world),
 *     since the array lives on this GPU only and cannot be shared with
 *     other processes; args->ws is not read;
 *   - world * lse_merge_cp_workspace_bytes(...) must fit in the array,
 *     else LSE_MERGE_ESCRATCH is returned and nothing is launched;
 *   - each call first clears the workspace headers on `stream` (a memset,
 *     no allocation), so every call starts from zero and a wait that ran out
 *     in an earlier call needs no restart; the received rows need no
 *     clearing, every one is written before it is read;
 *   - all calls on a GPU share the one array: calls whose work overlaps on
 *     the GPU (different streams, no ordering between them) race and give
 *     wrong results; order them on one stream;
 *   - the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it for
 *     that device's current context (a new context, e.g. after
 *     cudaDeviceReset, looks it up again); make that first call before any
 *     stream capture begins.
 * A wait that runs out sets the status word of that rank's workspace inside
 * the array and the rank's outputs are left unwritten; the kernel still
 * returns.  Read the status words with lse_merge_cp_noalloc_status.
 * Returns the codes of lse_merge_cp_exchange_merge, LSE_MERGE_ESCRATCH, and
 * LSE_MERGE_ECUDA when the address look-up or the header clearing fails. */
#define LSE_MERGE_CP_NOALLOC_SCRATCH_BYTES (16 << 20)
int lse_merge_cp_exchange_merge_noalloc(const lse_merge_cp_args* args, lse_merge_stream_t stream);

/* The status words of the last lse_merge_cp_exchange_merge_noalloc call on
 * the current device: status[q], for every rank q < args->world, is 0 when
 * all of rank q's waits completed (its outputs were written), else bit s is
 * set for each sender s whose rows never landed (rank q's outputs were not
 * written).  `args` must describe that call (world, B, H, D and in_dtype
 * fix where each rank's workspace lies in the array; the pointers are not
 * read).  Like lse_merge_cp_status it first waits for all work on the
 * current device, on every stream, then copies the words to the host; it
 * allocates nothing.  Returns LSE_MERGE_ENULL, the size codes of
 * lse_merge_cp_exchange_merge_noalloc (EDIMS, EALIGN, ESCRATCH), or
 * LSE_MERGE_ECUDA when a CUDA call fails.  No counterpart on the pages. */
int lse_merge_cp_noalloc_status(const lse_merge_cp_args* args, uint32_t* status);

/* ---------------------------------------------------------------------------
 * The merge of partials that live in host memory.  (No counterpart on the
 * pages, whose merge reads device memory; it serves callers whose partials
 * arrive in host memory, and it is what an end-to-end measurement times.)
 *
 * A host context, made on the current device by lse_merge_host_create, owns
 * a device staging area of `stage_bytes` (cudaMalloc), three streams and
 * their events; lse_merge_host_destroy waits for its last call and frees it
 * all.  These two are set-up calls: they allocate and synchronise.
 *
 * lse_merge_host merges h_partial_o / h_partial_lse, in host memory (pinned,
 * e.g. cudaMallocHost, for full copy speed; pageable memory works but the
 * copies then stall the host), into h_out_o [B,H,D] of out_dtype and
 * h_out_lse [B,H] fp32 in host memory.  The partials are dense in one of two
 * layouts: LSE_MERGE_LAYOUT_BHRD (o [B,H,R,D], lse [B,H,R]) or
 * LSE_MERGE_LAYOUT_RBHD (o [R,B,H,D], lse [R,B,H]).  The batch is cut into
 * `chunks` slices along B (at most LSE_MERGE_HOST_MAX_CHUNKS); slice i is
 * copied to the staging area while slice i-1 is merged (lse_merge, one
 * kernel launch) and slice i-2's results are copied back, so the upload of
 * the partials bounds the call.  The call only enqueues: `stream` is made to
 * wait for the last copy back, so synchronising `stream` makes the host
 * outputs valid.  Unless flags has LSE_MERGE_HOST_PIPELINE, the uploads first
 * wait for the work already on `stream` and for the context's previous call
 * to finish; with it, when the previous call had the same sizes, slice i
 * waits only until the previous call has merged slice i (for a stream of
 * batches: the uploads then follow each other back to back), so the host
 * inputs must not be written by device work still pending on `stream`.  One
 * thread at a time per context; not for stream capture.
 *
 * lse_merge_host_stage_bytes gives the staging bytes a call of these sizes
 * needs.  Returns the codes of lse_merge, LSE_MERGE_ESCRATCH when the
 * context's staging area is too small, LSE_MERGE_EDEVICE when another device
 * is current, and LSE_MERGE_ECUDA when a CUDA call fails. */
#define LSE_MERGE_LAYOUT_BHRD 0
#define LSE_MERGE_LAYOUT_RBHD 1
#define LSE_MERGE_HOST_MAX_CHUNKS 64
#define LSE_MERGE_HOST_PIPELINE 1
typedef struct lse_merge_host_ctx lse_merge_host_ctx;
int lse_merge_host_stage_bytes(int R, int B, int H, int D, int in_dtype, int out_dtype,
                               int64_t* bytes);
int lse_merge_host_create(int64_t stage_bytes, lse_merge_host_ctx** ctx);
int lse_merge_host_destroy(lse_merge_host_ctx* ctx);
int lse_merge_host(lse_merge_host_ctx* ctx, const void* h_partial_o, const float* h_partial_lse,
                   int R, int B, int H, int D, int layout, int in_dtype, int out_dtype,
                   void* h_out_o, float* h_out_lse, int chunks, int flags,
                   lse_merge_stream_t stream);

/* A static, human-readable description of a return code. */
const char* lse_merge_strerror(int code);

/* The cudaError_t of the last failed launch on this host thread (0 if none). */
int lse_merge_last_cuda_error(void);

/* ABI version of this header; bumped on any incompatible change. */
int lse_merge_version(void);

#define LSE_MERGE_ABI_VERSION 4

#ifdef __cplusplus
}
#endif

#endif /* LSE_MERGE_H */
