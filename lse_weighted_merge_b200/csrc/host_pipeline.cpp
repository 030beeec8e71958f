// host_pipeline.cpp -- the merge of partials that live in host memory.
//
// A host context (lse_merge_host_create) owns, on one device, a staging
// area in device memory, three streams (uploads, merges, copies back) and
// per-chunk events.  lse_merge_host cuts the batch into chunks along B and
// enqueues, for chunk i: the copy of its partials (and their lse) from host
// memory into the staging area, the merge of the chunk (lse_merge on the
// staged copy), and the copy of the chunk's results back to host memory.
// Chunk i's upload overlaps chunk i-1's merge and chunk i-2's copy back, so
// the upload of the partials -- the only large transfer -- bounds the call.
// Calls on one context are ordered through the events: chunk i of a call
// reuses chunk i's staging bytes only after the previous call has merged
// them and copied their results back.
//
// Everything here is host code on the CUDA runtime: copies, events, stream
// waits and the merge's own launch.  Only lse_merge_host_create allocates.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>

#include "lse_merge.h"
#include "plan.h"

namespace lsem {
namespace {

constexpr int kMaxChunks = LSE_MERGE_HOST_MAX_CHUNKS;

struct ChunkEvents {
    cudaEvent_t landed, merged, copied;
};

}  // namespace
}  // namespace lsem

struct lse_merge_host_ctx {
    int device;
    char* stage;                 // device staging area
    int64_t stage_bytes;
    cudaStream_t s_in, s_merge, s_back;
    cudaEvent_t caller;          // the caller's stream, recorded at a call's start
    cudaEvent_t done;            // a call's last copy back
    lsem::ChunkEvents ev[2][lsem::kMaxChunks];
    int parity;                  // event set of the last call
    // geometry of the last call (a pipelined call reuses its chunk events
    // only when it cuts the batch the same way)
    int last_n;
    int64_t last_nb, last_key[8];
};

namespace lsem {
namespace {

int64_t up256(int64_t x) { return (x + 255) / 256 * 256; }

// Staging offsets of one call: partials, lse, outputs, merged lse.
struct Stage {
    int64_t o, l, out, out_l, total;
};

Stage stage_layout(int R, int B, int H, int D, int ib, int ob) {
    Stage s;
    s.o = 0;
    s.l = up256((int64_t)R * B * H * D * ib);
    s.out = s.l + up256((int64_t)R * B * H * 4);
    s.out_l = s.out + up256((int64_t)B * H * D * ob);
    s.total = s.out_l + up256((int64_t)B * H * 4);
    return s;
}

int fail(int code, cudaError_t e) {
    set_last_cuda_error((int)e);
    (void)cudaGetLastError();
    return code;
}

void destroy(lse_merge_host_ctx* c) {
    if (!c) return;
    for (int p = 0; p < 2; ++p)
        for (int i = 0; i < kMaxChunks; ++i) {
            if (c->ev[p][i].landed) cudaEventDestroy(c->ev[p][i].landed);
            if (c->ev[p][i].merged) cudaEventDestroy(c->ev[p][i].merged);
            if (c->ev[p][i].copied) cudaEventDestroy(c->ev[p][i].copied);
        }
    if (c->caller) cudaEventDestroy(c->caller);
    if (c->done) cudaEventDestroy(c->done);
    if (c->s_in) cudaStreamDestroy(c->s_in);
    if (c->s_merge) cudaStreamDestroy(c->s_merge);
    if (c->s_back) cudaStreamDestroy(c->s_back);
    if (c->stage) cudaFree(c->stage);
    delete c;
}

}  // namespace
}  // namespace lsem

extern "C" {

int lse_merge_host_stage_bytes(int R, int B, int H, int D, int in_dtype, int out_dtype,
                               int64_t* bytes) {
    if (!bytes) return LSE_MERGE_ENULL;
    const int ib = lsem::elem_bytes(in_dtype), ob = lsem::elem_bytes(out_dtype);
    if (ib == 0 || ob == 0) return LSE_MERGE_EDTYPE;
    if (R < 1 || B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    if ((__int128)R * B * H * D * ib > ((__int128)1 << 60)) return LSE_MERGE_EDIMS;
    *bytes = lsem::stage_layout(R, B, H, D, ib, ob).total;
    return LSE_MERGE_OK;
}

int lse_merge_host_create(int64_t stage_bytes, lse_merge_host_ctx** ctx) {
    using namespace lsem;
    if (!ctx) return LSE_MERGE_ENULL;
    if (stage_bytes < 256) return LSE_MERGE_EDIMS;
    lse_merge_host_ctx* c = new (std::nothrow) lse_merge_host_ctx();
    if (!c) return LSE_MERGE_ECUDA;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess) e = cudaMalloc(&c->stage, (size_t)stage_bytes);
    c->stage_bytes = stage_bytes;
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->s_merge, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->s_back, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->caller, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->done, cudaEventDisableTiming);
    for (int p = 0; p < 2 && e == cudaSuccess; ++p)
        for (int i = 0; i < kMaxChunks && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&c->ev[p][i].landed, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev[p][i].merged, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev[p][i].copied, cudaEventDisableTiming);
        }
    if (e == cudaSuccess) e = cudaEventRecord(c->done, c->s_back);   // nothing pending yet
    if (e != cudaSuccess) {
        destroy(c);
        return fail(LSE_MERGE_ECUDA, e);
    }
    c->last_n = 0;
    *ctx = c;
    return LSE_MERGE_OK;
}

int lse_merge_host_destroy(lse_merge_host_ctx* ctx) {
    if (!ctx) return LSE_MERGE_ENULL;
    const cudaError_t e = cudaStreamSynchronize(ctx->s_back);   // the last call's copies back
    (void)cudaStreamSynchronize(ctx->s_merge);
    (void)cudaStreamSynchronize(ctx->s_in);
    lsem::destroy(ctx);
    if (e != cudaSuccess) return lsem::fail(LSE_MERGE_ECUDA, e);
    return LSE_MERGE_OK;
}

int lse_merge_host(lse_merge_host_ctx* c, const void* h_partial_o, const float* h_partial_lse,
                   int R, int B, int H, int D, int layout, int in_dtype, int out_dtype,
                   void* h_out_o, float* h_out_lse, int chunks, int flags,
                   lse_merge_stream_t stream) {
    using namespace lsem;
    if (!c || !h_partial_o || !h_partial_lse || !h_out_o || !h_out_lse) return LSE_MERGE_ENULL;
    const int ib = elem_bytes(in_dtype), ob = elem_bytes(out_dtype);
    if (ib == 0 || ob == 0) return LSE_MERGE_EDTYPE;
    if (R < 1 || B < 1 || H < 1 || D < 1 || chunks < 1) return LSE_MERGE_EDIMS;
    if (layout != LSE_MERGE_LAYOUT_BHRD && layout != LSE_MERGE_LAYOUT_RBHD) return LSE_MERGE_ESTRIDE;
    if (flags & ~LSE_MERGE_HOST_PIPELINE) return LSE_MERGE_EDIMS;
    int64_t need = 0;
    int rc = lse_merge_host_stage_bytes(R, B, H, D, in_dtype, out_dtype, &need);
    if (rc != LSE_MERGE_OK) return rc;
    if (need > c->stage_bytes) return LSE_MERGE_ESCRATCH;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(LSE_MERGE_ECUDA, e);
    if (dev != c->device) return LSE_MERGE_EDEVICE;
    const Stage st = stage_layout(R, B, H, D, ib, ob);
    char* d_o = c->stage + st.o;
    float* d_l = reinterpret_cast<float*>(c->stage + st.l);
    char* d_out = c->stage + st.out;
    float* d_out_l = reinterpret_cast<float*>(c->stage + st.out_l);

    const int64_t nb = (B + (int64_t)chunks - 1) / chunks;   // batches per chunk
    const int n = (int)((B + nb - 1) / nb);
    if (n > kMaxChunks) return LSE_MERGE_EDIMS;
    const cudaStream_t caller = reinterpret_cast<cudaStream_t>(stream);
    const int64_t key[8] = {R, B, H, D, layout, in_dtype, out_dtype, nb};
    const bool reuse = (flags & LSE_MERGE_HOST_PIPELINE) && c->last_n == n && c->last_nb == nb &&
                       std::memcmp(key, c->last_key, sizeof key) == 0;
    const ChunkEvents* prev = c->ev[c->parity];
    const int par = c->parity ^ 1;
    ChunkEvents* cur = c->ev[par];

#define LSEM_TRY(x)                                   \
    do {                                              \
        e = (x);                                      \
        if (e != cudaSuccess) return fail(LSE_MERGE_ECUDA, e); \
    } while (0)

    LSEM_TRY(cudaEventRecord(c->caller, caller));
    if (!reuse) {
        // The whole staging area is free once the previous call's last copy
        // back is done; the host buffers may still be in use on the caller's
        // stream.
        LSEM_TRY(cudaStreamWaitEvent(c->s_in, c->done, 0));
        LSEM_TRY(cudaStreamWaitEvent(c->s_in, c->caller, 0));
        LSEM_TRY(cudaStreamWaitEvent(c->s_back, c->done, 0));
    }
    // the host outputs may be in use on the caller's stream
    LSEM_TRY(cudaStreamWaitEvent(c->s_back, c->caller, 0));

    const int64_t row_o = (int64_t)H * D * ib;        // one batch of one partial plane
    const int64_t row_l = (int64_t)H * 4;
    for (int i = 0; i < n; ++i) {
        const int64_t b0 = (int64_t)i * nb, b1 = b0 + nb < B ? b0 + nb : B, nbi = b1 - b0;
        // ---- upload chunk i
        if (reuse) LSEM_TRY(cudaStreamWaitEvent(c->s_in, prev[i].merged, 0));
        if (layout == LSE_MERGE_LAYOUT_BHRD) {   // [B,H,R,D]: one contiguous block per chunk
            LSEM_TRY(cudaMemcpyAsync(d_o + b0 * R * row_o, static_cast<const char*>(h_partial_o) + b0 * R * row_o,
                                     (size_t)(nbi * R * row_o), cudaMemcpyHostToDevice, c->s_in));
            LSEM_TRY(cudaMemcpyAsync(d_l + b0 * R * H, h_partial_lse + b0 * R * H,
                                     (size_t)(nbi * R * row_l), cudaMemcpyHostToDevice, c->s_in));
        } else {                                 // [R,B,H,D]: R blocks, one per partial plane
            LSEM_TRY(cudaMemcpy2DAsync(d_o + b0 * row_o, (size_t)(B * row_o),
                                       static_cast<const char*>(h_partial_o) + b0 * row_o,
                                       (size_t)(B * row_o), (size_t)(nbi * row_o), (size_t)R,
                                       cudaMemcpyHostToDevice, c->s_in));
            LSEM_TRY(cudaMemcpy2DAsync(d_l + b0 * H, (size_t)(B * row_l), h_partial_lse + b0 * H,
                                       (size_t)(B * row_l), (size_t)(nbi * row_l), (size_t)R,
                                       cudaMemcpyHostToDevice, c->s_in));
        }
        LSEM_TRY(cudaEventRecord(cur[i].landed, c->s_in));
        // ---- merge chunk i (its outputs' staging is free once the previous
        // call copied them back)
        LSEM_TRY(cudaStreamWaitEvent(c->s_merge, cur[i].landed, 0));
        if (reuse) LSEM_TRY(cudaStreamWaitEvent(c->s_merge, prev[i].copied, 0));
        lse_merge_strides s;
        const void* po;
        const float* pl;
        if (layout == LSE_MERGE_LAYOUT_BHRD) {
            s.o_r = D;
            s.o_b = (int64_t)H * R * D;
            s.o_h = (int64_t)R * D;
            s.lse_r = 1;
            s.lse_b = (int64_t)H * R;
            s.lse_h = R;
            po = d_o + b0 * R * row_o;
            pl = d_l + b0 * R * H;
        } else {
            s.o_r = (int64_t)B * H * D;
            s.o_b = (int64_t)H * D;
            s.o_h = D;
            s.lse_r = (int64_t)B * H;
            s.lse_b = H;
            s.lse_h = 1;
            po = d_o + b0 * row_o;
            pl = d_l + b0 * H;
        }
        rc = lse_merge(po, pl, R, (int)nbi, H, D, &s, in_dtype, out_dtype,
                       d_out + b0 * H * D * ob, d_out_l + b0 * H, c->s_merge);
        if (rc != LSE_MERGE_OK) return rc;
        LSEM_TRY(cudaEventRecord(cur[i].merged, c->s_merge));
        // ---- copy chunk i's results back
        LSEM_TRY(cudaStreamWaitEvent(c->s_back, cur[i].merged, 0));
        LSEM_TRY(cudaMemcpyAsync(static_cast<char*>(h_out_o) + b0 * H * D * ob, d_out + b0 * H * D * ob,
                                 (size_t)(nbi * H * D * ob), cudaMemcpyDeviceToHost, c->s_back));
        LSEM_TRY(cudaMemcpyAsync(h_out_lse + b0 * H, d_out_l + b0 * H, (size_t)(nbi * H * 4),
                                 cudaMemcpyDeviceToHost, c->s_back));
        LSEM_TRY(cudaEventRecord(cur[i].copied, c->s_back));
    }
    LSEM_TRY(cudaEventRecord(c->done, c->s_back));
    LSEM_TRY(cudaStreamWaitEvent(caller, c->done, 0));
#undef LSEM_TRY
    c->parity = par;
    c->last_n = n;
    c->last_nb = nb;
    std::memcpy(c->last_key, key, sizeof key);
    return LSE_MERGE_OK;
}

}  // extern "C"
