// cp_exchange.cu -- context-parallel exchange and merge in one kernel (sm_100a).
//
// Under context-parallel decode every rank holds the partials (o, lse) of its
// own KV shard for all heads; the heads are then scattered so that each rank
// merges the partials of the heads it owns (page "[flashinfer] FlashInfer의
// Context-Parallel Decode 최적화: Fused A2A + LSE Reduce", section "들어가며"
// for the partials; section "코드 분석 / 1. Fused Kernel 구현" for the fused
// design in which the ranks write straight into the owner's buffer over
// NVLink and the owner merges once everything has landed).
//
// One launch, per rank `me` (blockIdx.y picks the rank among those the launch
// plays; blockIdx.x is the CTA within the rank):
//   1. send: the rank's partial rows of heads owned by rank q != me are
//      copied, 16 bytes per thread and step, into q's workspace (the slot of
//      sender me; parity e & 1 across GPUs, always slot 0 when one launch
//      plays every rank).  Each CTA owns a contiguous range of the
//      (q, b, head, 16-byte column) units, so consecutive threads write
//      consecutive addresses of one receiver;
//   2. land: after a CTA barrier, one thread makes the CTA's stores visible
//      (system scope; device scope when every rank is in this launch, so all
//      readers are on this GPU) and adds the number of units the CTA sent to
//      q to q's landed counter of sender me.  The count does not depend on
//      how many CTAs the sender used, so ranks may launch different grids;
//   3. wait: lane s of warp 0 of every CTA polls sender s's landed counter in
//      me's workspace (acquire, same scope) until it reached e * U units (e:
//      the number of this call, kept in the workspace header), all senders
//      at once, bounded by the GPU global timer and by a poll count.  A wait
//      that runs out sets the sender's bit in me's status word and the CTA
//      skips its merge;
//   4. merge: each thread merges one 16-byte column of one owned row over all
//      senders: its own partial read in place from local_o, the others from
//      the workspace (L2-only loads, since other SMs or GPUs wrote them during
//      this launch), fp32 accumulation, one reciprocal, conversion.
// The call number e comes from a count of arriving CTAs kept in the rank's
// workspace, so the next call (or the next replay of a captured graph) is
// call e + 1 without the host passing anything.
// All CTAs of the launch are co-resident (cooperative launch), so a CTA that
// waits never keeps a sending CTA of the same launch from running.
//
// The peer traffic is plain 16-byte stores and one atomic add per CTA and
// receiver; no load reads another GPU's memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "lse_merge.h"
#include "plan.h"

namespace lsem {
namespace {

constexpr int kMaxWorld = LSE_MERGE_CP_MAX_WORLD;
// 16-byte units in flight per thread while sending: kSendShallow when each
// thread sends at most that many, else kSendDeep (measured on B200, every
// rank in one launch, graph-replayed: 8 ranks x B=256 H=64 D=128 took
// 21.5 us at 8 against 22.8 us at 4; 2 ranks x B=1 H=2 D=64 took 3.5 us at
// 4 against 3.7 us at 8).
constexpr int kSendShallow = 4;
constexpr int kSendDeep = 8;
// Poll back-off of the landed-counter wait (measured on B200 with every rank
// in one launch: 32..256 ns gave 4.43 us per call for 2 ranks of one head,
// 64..2048 ns 4.53 us).
constexpr unsigned kSleepMinNs = 32;
constexpr unsigned kSleepMaxNs = 256;
constexpr unsigned kFullMask = 0xffffffffu;
// Threads per CTA: kCpBlock = 256 (measured on B200 for 2 ranks of one head:
// 128 threads 5.66 us against 4.43 us; a 64-register cap, 4 CTAs per SM,
// 6.15 us).
constexpr int kThreads = kCpBlock;

// Workspace header (kCpHeaderBytes): at 8*s the landed counter of sender s
// (u64: 16-byte units received from s over all calls); the status word at
// LSE_MERGE_CP_STATUS_OFFSET; at kArrivedOffset, on a cache line apart from
// the landed counters (which take other ranks' atomics and polls), the
// rank's CTA arrival count: kCallShares per call.
constexpr int64_t kArrivedOffset = 128;
constexpr unsigned long long kCallShares = 1ull << 20;   // > any grid: every share >= 1

struct CpParams {
    const char* local_o[kMaxWorld];   // per played rank, dense [B, H, D]
    const float* local_lse[kMaxWorld];
    char* out_o[kMaxWorld];           // per played rank, dense [B, Hq, D]
    float* out_lse[kMaxWorld];
    char* ws[kMaxWorld];              // every rank's workspace
    int world, rank_begin, H, Hq;
    uint32_t dv;                      // 16-byte units per row
    int64_t U;                        // units per (sender, receiver) pair
    int64_t rowbytes;                 // D * in_bytes
    int64_t slot_o, slot_l, o_off, l_off;
    int64_t timeout_ns, max_polls;
    int64_t chunk;                    // send units per CTA
    unsigned long long share, share0; // arrival shares: CTA 0 share0, the others share
    int local;                        // every rank is played by this launch (one GPU)
    int silent;                       // a rank that sends nothing (test flag), else -1
    uint64_t c_U, c_dv, c_Hq;         // fastdiv constants of U, dv and Hq
};

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned long long ld_acquire_sys(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Loads of data written during this launch by other SMs or GPUs: cached in
// L2 only (L1 is not coherent), 256-byte L2 prefetch for the row's neighbours.
__device__ __forceinline__ uint4 ld_cg16(const char* p) {
    uint4 v;
    asm volatile("ld.global.cg.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}
__device__ __forceinline__ float ld_cg_f32(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}

// n / d and n % d by the 32-bit constant division: the planner keeps every
// unit index below 2^31.
__device__ __forceinline__ void divmod(int64_t n, uint64_t c, int64_t d, int64_t& q, int64_t& r) {
    const uint32_t qq = fastdiv((uint32_t)n, c, (uint32_t)d);
    q = qq;
    r = (int64_t)((uint32_t)n - qq * (uint32_t)d);
}

// UNROLL units of one sending thread: units u, u + kThreads, ... .
template <int UNROLL>
struct SendBatch {
    uint4 x[UNROLL];
    float lv[UNROLL];
    int64_t rem[UNROLL];   // unit index inside the receiver's block
    int64_t row[UNROLL];   // row (b * Hq + head) inside the receiver's block
    int q[UNROLL];         // receiver, or -1 past the CTA's range
};

// Load the partial columns (and, for a row's first column, the lse) of the
// batch at u; nothing here depends on the call number.
template <int UNROLL>
__device__ __forceinline__ void load_batch(const CpParams& p, int me, int64_t u, int64_t u1,
                                           const char* src_o, const float* src_l,
                                           SendBatch<UNROLL>& sb) {
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
        const int64_t uk = u + (int64_t)k * kThreads;
        sb.q[k] = -1;
        sb.lv[k] = 0.f;
        sb.rem[k] = 0;
        sb.row[k] = 0;
        sb.x[k] = make_uint4(0u, 0u, 0u, 0u);
        if (uk < u1) {
            int64_t qi, rem, row, v, b, hq;
            divmod(uk, p.c_U, p.U, qi, rem);
            divmod(rem, p.c_dv, p.dv, row, v);
            divmod(row, p.c_Hq, p.Hq, b, hq);
            const int q = (int)qi + ((int)qi >= me ? 1 : 0);   // receiver
            const int64_t srow = b * p.H + (int64_t)q * p.Hq + hq;
            sb.x[k] = ld_stream16(src_o + srow * p.rowbytes + v * 16);
            if (v == 0) sb.lv[k] = __ldg(src_l + srow);
            sb.q[k] = q;
            sb.rem[k] = rem;
            sb.row[k] = v == 0 ? row : -1;
        }
    }
}

// Store the batch into the receivers' slots of sender me, parity par.
template <int UNROLL>
__device__ __forceinline__ void store_batch(const CpParams& p, int me, int w1, int par,
                                            const SendBatch<UNROLL>& sb) {
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
        const int q = sb.q[k];
        if (q < 0) continue;
        const int slot = me - (me > q ? 1 : 0);   // sender slot at q
        const int64_t blk = (int64_t)par * w1 + slot;
        *reinterpret_cast<uint4*>(p.ws[q] + p.o_off + blk * p.slot_o + sb.rem[k] * 16) = sb.x[k];
        if (sb.row[k] >= 0)
            reinterpret_cast<float*>(p.ws[q] + p.l_off + blk * p.slot_l)[sb.row[k]] = sb.lv[k];
    }
}

template <typename TIn, typename TOut, int UNROLL>
__global__ void __launch_bounds__(kThreads, 2) cp_exchange_merge_kernel(const __grid_constant__ CpParams p) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    const int pr = blockIdx.y;
    const int me = p.rank_begin + pr;
    const int w1 = p.world - 1;
    const int64_t cta = blockIdx.x;
    const char* src_o = p.local_o[pr];
    const float* src_l = p.local_lse[pr];
    char* const mine = p.ws[me];
    // This call's number e (1 for the first call after the workspace was
    // zeroed): on arrival CTA c adds its share of kCallShares to the rank's
    // arrival count (shares of one call sum to kCallShares whatever the
    // grid), and calls of one rank are stream-ordered, so the count a CTA of
    // call e gets back lies in [(e-1)*kCallShares, e*kCallShares).  The
    // atomic's round trip overlaps the first partial loads.
    __shared__ unsigned long long s_e;
    unsigned long long arrived = 0;
    if (threadIdx.x == 0)
        arrived = atomicAdd(reinterpret_cast<unsigned long long*>(mine + kArrivedOffset),
                            cta == 0 ? p.share0 : p.share);

    // ---- 1. send the rows other ranks own: CTA c sends units
    // [c*chunk, (c+1)*chunk) of the rank's total.
    const int64_t total = (int64_t)w1 * p.U;
    const int64_t u0 = min(total, cta * p.chunk);
    const int64_t u1 = me == p.silent ? u0 : min(total, u0 + p.chunk);
    int64_t u = u0 + threadIdx.x;
    SendBatch<UNROLL> sb;
    load_batch(p, me, u, u1, src_o, src_l, sb);
    // Receive slot of this call.  Ranks on different GPUs alternate two slots
    // by the parity of e, so a rank may start call e + 1 while a peer still
    // reads call e.  When this launch plays every rank, call e + 1 cannot
    // start before call e has ended, one slot suffices, and the stores need
    // not wait for e.
    int par = 0;
    if (!p.local) {
        if (threadIdx.x == 0) s_e = arrived / kCallShares + 1;
        __syncthreads();
        par = (int)(s_e & 1);
    }
    for (;;) {
        store_batch(p, me, w1, par, sb);
        u += (int64_t)kThreads * UNROLL;
        if (u >= u1) break;
        load_batch(p, me, u, u1, src_o, src_l, sb);
    }
    if (p.local && threadIdx.x == 0) s_e = arrived / kCallShares + 1;

    // ---- 2. land: publish this CTA's units to each receiver
    __syncthreads();
    const unsigned long long e = s_e;
    if (threadIdx.x == 0 && u1 > u0) {
        // Every rank on this GPU: device scope orders the stores for all
        // readers; otherwise the readers are other GPUs and need system scope.
        if (p.local) __threadfence();
        else __threadfence_system();
        for (int qi = 0; qi < w1; ++qi) {
            const int64_t lo = max(u0, (int64_t)qi * p.U), hi = min(u1, (int64_t)(qi + 1) * p.U);
            if (hi > lo) {
                const int q = qi + (qi >= me ? 1 : 0);
                unsigned long long* c = reinterpret_cast<unsigned long long*>(p.ws[q]) + me;
                if (p.local) atomicAdd(c, (unsigned long long)(hi - lo));
                else atomicAdd_system(c, (unsigned long long)(hi - lo));
            }
        }
    }

    // ---- 3. wait until every sender's units of calls 1..e have landed here (bounded)
    // Lane s of warp 0 polls sender s's counter, so the waits for all senders
    // overlap instead of costing one memory round trip each.
    __shared__ int s_ok;
    const unsigned long long target = e * (unsigned long long)p.U;
    if (threadIdx.x < 32) {
        const int s = threadIdx.x;
        const unsigned long long* landed = reinterpret_cast<const unsigned long long*>(mine) + s;
        bool ok = s >= p.world || s == me;
        int64_t polls = 0;
        unsigned ns = kSleepMinNs;
        const uint64_t t0 = global_ns();
        for (;;) {
            if (!ok) ok = (p.local ? ld_acquire_gpu(landed) : ld_acquire_sys(landed)) >= target;
            if (__all_sync(kFullMask, ok)) break;
            if (++polls > p.max_polls || global_ns() - t0 > (uint64_t)p.timeout_ns) break;
            __nanosleep(ns);
            if (ns < kSleepMaxNs) ns <<= 1;
        }
        const unsigned missing = __ballot_sync(kFullMask, !ok);   // bit s: sender s
        if (s == 0) {
            if (missing) atomicOr(reinterpret_cast<unsigned*>(mine + LSE_MERGE_CP_STATUS_OFFSET), missing);
            s_ok = missing == 0;
        }
    }
    __syncthreads();

    // ---- 4. merge the owned rows over all senders (skipped after a timeout)
    // A thread takes units w and w + stride together: the loads of both go
    // out before either is merged, so twice as many are in flight.
    char* const dst_o = p.out_o[pr];
    float* const dst_l = p.out_lse[pr];
    const int64_t wend = s_ok ? p.U : 0;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    struct Unit {
        int64_t w, row, v;
        uint4 x[kMaxWorld];
        float l[kMaxWorld];
    };
    auto load_unit = [&](Unit& u) {
        int64_t b, hq;
        divmod(u.w, p.c_dv, p.dv, u.row, u.v);
        divmod(u.row, p.c_Hq, p.Hq, b, hq);
        const int64_t srow = b * p.H + (int64_t)me * p.Hq + hq;
#pragma unroll
        for (int s = 0; s < kMaxWorld; ++s) {
            u.x[s] = make_uint4(0u, 0u, 0u, 0u);
            u.l[s] = -INFINITY;
            if (s < p.world) {
                if (s == me) {
                    u.x[s] = ld_stream16(src_o + srow * p.rowbytes + u.v * 16);
                    u.l[s] = __ldg(src_l + srow);
                } else {
                    const int64_t blk = (int64_t)par * w1 + (s - (s > me ? 1 : 0));
                    u.x[s] = ld_cg16(mine + p.o_off + blk * p.slot_o + u.w * 16);
                    u.l[s] = ld_cg_f32(reinterpret_cast<const float*>(mine + p.l_off + blk * p.slot_l) + u.row);
                }
            }
        }
    };
    auto merge_unit = [&](const Unit& u) {
        float m = -INFINITY;
#pragma unroll
        for (int s = 0; s < kMaxWorld; ++s) m = fmaxf(m, u.l[s]);
        // An all-empty row has m = -inf; subtracting 0 keeps every weight
        // exp(-inf) = 0 instead of NaN.
        const float mref = (m == -INFINITY) ? 0.f : m;
        uint64_t acc[N2];
#pragma unroll
        for (int k = 0; k < N2; ++k) acc[k] = 0ull;
        float esum = 0.f;
#pragma unroll
        for (int s = 0; s < kMaxWorld; ++s) {
            const float e = expf(u.l[s] - mref);   // 0 for an empty partial or s >= world
            esum += e;
            if (e != 0.f) {                        // an empty partial's o (maybe NaN) is not read
                uint64_t xx[N2];
                Elem<TIn>::unpack2(u.x[s], xx);
                const uint64_t ww = pack2f(e, e);
#pragma unroll
                for (int k = 0; k < N2; ++k) fma2(acc[k], xx[k], ww);
            }
        }
        const float inv = esum > 0.f ? 1.f / esum : 0.f;
        float f[N];
#pragma unroll
        for (int k = 0; k < N2; ++k) {
            unpack2f(acc[k], f[2 * k], f[2 * k + 1]);
            f[2 * k] *= inv;
            f[2 * k + 1] *= inv;
        }
        store_vec<TOut, N>(dst_o + u.w * N * (int64_t)sizeof(TOut), f);
        if (u.v == 0) dst_l[u.row] = esum > 0.f ? m + logf(esum) : -INFINITY;
    };
    for (int64_t w = cta * kThreads + threadIdx.x; w < wend; w += 2 * stride) {
        Unit a, b;
        a.w = w;
        b.w = w + stride;
        load_unit(a);
        const bool two = b.w < wend;
        if (two) load_unit(b);
        merge_unit(a);
        if (two) merge_unit(b);
    }
}

using CpFn = void (*)(CpParams);

template <typename TIn, int UNROLL>
CpFn pick_out(int out_dtype) {
    switch (out_dtype) {
        case LSE_MERGE_F32: return cp_exchange_merge_kernel<TIn, float, UNROLL>;
        case LSE_MERGE_F16: return cp_exchange_merge_kernel<TIn, __half, UNROLL>;
        default: return cp_exchange_merge_kernel<TIn, __nv_bfloat16, UNROLL>;
    }
}

template <int UNROLL>
CpFn pick_cp(int in_dtype, int out_dtype) {
    switch (in_dtype) {
        case LSE_MERGE_F32: return pick_out<float, UNROLL>(out_dtype);
        case LSE_MERGE_F16: return pick_out<__half, UNROLL>(out_dtype);
        default: return pick_out<__nv_bfloat16, UNROLL>(out_dtype);
    }
}

// Co-resident CTAs per SM and SM count, cached per (kernel, device).
struct CoEntry {
    const void* fn;
    int dev, per_sm, sms;
};
constexpr int kCoSlots = 64;
CoEntry g_co[kCoSlots];
int g_co_n = 0;
std::mutex g_co_mu;

int co_resident(const void* fn, int64_t* capacity) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    {
        std::lock_guard<std::mutex> lk(g_co_mu);
        for (int i = 0; i < g_co_n; ++i)
            if (g_co[i].fn == fn && g_co[i].dev == dev) {
                *capacity = (int64_t)g_co[i].per_sm * g_co[i].sms;
                return 0;
            }
    }
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0);
    if (e != cudaSuccess) return (int)e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return (int)e;
    {
        std::lock_guard<std::mutex> lk(g_co_mu);
        if (g_co_n < kCoSlots) g_co[g_co_n++] = CoEntry{fn, dev, per_sm, sms};
    }
    *capacity = (int64_t)per_sm * sms;
    return 0;
}

int fail_cuda(int code, int e) {
    set_last_cuda_error(e);
    (void)cudaGetLastError();   // the failure belongs to this call; do not leave it pending
    return code;
}

static_assert(sizeof(cudaIpcMemHandle_t) == LSE_MERGE_CP_IPC_HANDLE_BYTES, "IPC handle size");

}  // namespace
}  // namespace lsem

extern "C" {

int lse_merge_cp_exchange_merge(const lse_merge_cp_args* a, lse_merge_stream_t stream) {
    using namespace lsem;
    if (!a) return LSE_MERGE_ENULL;
    CpPlan pl;
    const int rc = make_cp_plan(*a, &pl);
    if (rc != LSE_MERGE_OK) return rc;

    CpParams kp{};
    for (int i = 0; i < a->rank_count; ++i) {
        kp.local_o[i] = static_cast<const char*>(a->local_o[i]);
        kp.local_lse[i] = a->local_lse[i];
        kp.out_o[i] = static_cast<char*>(a->out_o[i]);
        kp.out_lse[i] = a->out_lse[i];
    }
    for (int q = 0; q < a->world; ++q) kp.ws[q] = static_cast<char*>(a->ws[q]);
    kp.world = a->world;
    kp.rank_begin = a->rank_begin;
    kp.H = a->H;
    kp.Hq = pl.Hq;
    kp.dv = (uint32_t)pl.dv;
    kp.U = pl.U;
    kp.rowbytes = (int64_t)a->D * pl.in_bytes;
    kp.slot_o = pl.slot_o;
    kp.slot_l = pl.slot_l;
    kp.o_off = pl.o_off;
    kp.l_off = pl.l_off;
    kp.timeout_ns = a->timeout_ns;
    // Second bound on the wait, should the global timer not advance: with
    // sleeps growing to ~2 us, this many polls take several times the timeout.
    kp.max_polls = a->timeout_ns / 256 + 1024;
    const int64_t send_units = (int64_t)(a->world - 1) * pl.U;
    kp.local = a->rank_count == a->world && !(a->flags & LSE_MERGE_CP_FLAG_CROSS_GPU_PROTOCOL);
    kp.silent = (a->flags & LSE_MERGE_CP_FLAG_TEST_SILENT_LAST_RANK) ? a->world - 1 : -1;
    kp.c_U = fastdiv_c((uint32_t)pl.U);
    kp.c_dv = fastdiv_c(kp.dv);
    kp.c_Hq = fastdiv_c((uint32_t)pl.Hq);

    // One CTA per kThreads units of the larger phase, at most what is
    // co-resident; the deep send batch once a thread sends more units than
    // the shallow one holds.
    const int64_t work = send_units > pl.U ? send_units : pl.U;
    CpFn fn = nullptr;
    int64_t ctas = 0;
    for (int deep = 0; deep < 2; ++deep) {
        fn = deep ? pick_cp<kSendDeep>(a->in_dtype, a->out_dtype)
                  : pick_cp<kSendShallow>(a->in_dtype, a->out_dtype);
        int64_t capacity = 0;
        const int ce = co_resident((const void*)fn, &capacity);
        if (ce != 0) return fail_cuda(LSE_MERGE_ELAUNCH, ce);
        const int64_t cap = capacity / a->rank_count;
        if (cap < 1) return fail_cuda(LSE_MERGE_ELAUNCH, (int)cudaErrorCooperativeLaunchTooLarge);
        ctas = (work + kThreads - 1) / kThreads;
        if (ctas > cap) ctas = cap;
        if (ctas < 1) ctas = 1;
        kp.chunk = (send_units + ctas - 1) / ctas;
        if (kp.chunk <= (int64_t)kSendShallow * kThreads) break;
    }
    kp.share = kCallShares / (unsigned long long)ctas;
    kp.share0 = kCallShares - (unsigned long long)(ctas - 1) * kp.share;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ctas, (unsigned)a->rank_count, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fn, kp);
    if (e != cudaSuccess) return fail_cuda(LSE_MERGE_ELAUNCH, (int)e);
    return LSE_MERGE_OK;
}

int lse_merge_cp_workspace_create(int64_t bytes, void** ws) {
    if (!ws) return LSE_MERGE_ENULL;
    if (bytes < lsem::kCpHeaderBytes) return LSE_MERGE_EDIMS;
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, (size_t)bytes);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    e = cudaMemset(p, 0, (size_t)bytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        (void)cudaFree(p);
        return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    }
    *ws = p;
    return LSE_MERGE_OK;
}

int lse_merge_cp_status(const void* ws, uint32_t* status) {
    if (!ws || !status) return LSE_MERGE_ENULL;
    // every call already enqueued on the device, on any stream, first
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(status, static_cast<const char*>(ws) + LSE_MERGE_CP_STATUS_OFFSET,
                       sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return LSE_MERGE_OK;
}

int lse_merge_cp_workspace_zero(void* ws, int64_t bytes) {
    if (!ws) return LSE_MERGE_ENULL;
    if (bytes < lsem::kCpHeaderBytes) return LSE_MERGE_EDIMS;
    cudaError_t e = cudaDeviceSynchronize();   // no call of this device still uses it
    if (e == cudaSuccess) e = cudaMemset(ws, 0, (size_t)bytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return LSE_MERGE_OK;
}

int lse_merge_cp_workspace_destroy(void* ws) {
    if (!ws) return LSE_MERGE_ENULL;
    const cudaError_t e = cudaFree(ws);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return LSE_MERGE_OK;
}

int lse_merge_cp_ipc_handle(void* ws, void* handle) {
    if (!ws || !handle) return LSE_MERGE_ENULL;
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, ws);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    std::memcpy(handle, &h, sizeof(h));
    return LSE_MERGE_OK;
}

int lse_merge_cp_ipc_open(const void* handle, void** peer_ws) {
    if (!handle || !peer_ws) return LSE_MERGE_ENULL;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* p = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    *peer_ws = p;
    return LSE_MERGE_OK;
}

int lse_merge_cp_ipc_close(void* peer_ws) {
    if (!peer_ws) return LSE_MERGE_ENULL;
    const cudaError_t e = cudaIpcCloseMemHandle(peer_ws);
    if (e != cudaSuccess) return lsem::fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return LSE_MERGE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------
// The entry point that allocates nothing: its workspaces live in this array.
namespace lsem {
namespace {

constexpr int64_t kNoAllocBytes = LSE_MERGE_CP_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch, looked up once per device and
// context.  In host code the array's name is only a stand-in for the symbol,
// never an address a kernel may be given.  The address is kept with the id
// of the context it was looked up in (cuCtxGetId, reached through the
// runtime's driver entry points, so the library needs no libcuda link): a
// later context on the device (after cudaDeviceReset) looks it up again.
constexpr int kMaxDevices = 64;
struct NoAllocAddr {
    void* ptr;
    unsigned long long ctx_id;   // 0: unknown
};
NoAllocAddr g_noalloc[kMaxDevices] = {};
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = int (*)(void**);                    // cuCtxGetCurrent
using CtxGetIdFn = int (*)(void*, unsigned long long*);     // cuCtxGetId
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
bool g_ctx_fns_tried = false;

// Id of the current context, or 0 when it cannot be told.  Caller holds g_noalloc_mu.
unsigned long long current_ctx_id() {
    if (!g_ctx_fns_tried) {
        g_ctx_fns_tried = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<CtxGetIdFn>(f);
        (void)cudaGetLastError();
    }
    if (!g_ctx_current || !g_ctx_id) return 0;
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != 0 || !ctx || g_ctx_id(ctx, &id) != 0) return 0;
    return id;
}

int noalloc_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    const bool cacheable = dev >= 0 && dev < kMaxDevices;
    const unsigned long long id = current_ctx_id();
    if (cacheable && id != 0 && g_noalloc[dev].ptr && g_noalloc[dev].ctx_id == id) {
        *ptr = g_noalloc[dev].ptr;
        return 0;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return (int)e;
    // The look-up makes the device's primary context current if it was not.
    const unsigned long long id2 = id != 0 ? id : current_ctx_id();
    if (cacheable) g_noalloc[dev] = NoAllocAddr{p, id2};
    *ptr = p;
    return 0;
}

// Where each rank's workspace lies in the array for these sizes: every
// workspace starts on a 256-byte boundary, `pitch` bytes apart.
int noalloc_layout(const lse_merge_cp_args* args, int64_t* pitch) {
    int64_t ws_bytes = 0;
    const int rc = lse_merge_cp_workspace_bytes(args->world, args->B, args->H, args->D,
                                                args->in_dtype, &ws_bytes);
    if (rc != LSE_MERGE_OK) return rc;
    *pitch = (ws_bytes + 255) / 256 * 256;
    if ((int64_t)args->world * *pitch > kNoAllocBytes) return LSE_MERGE_ESCRATCH;
    return LSE_MERGE_OK;
}

}  // namespace
}  // namespace lsem

extern "C" int lse_merge_cp_exchange_merge_noalloc(const lse_merge_cp_args* args,
                                                   lse_merge_stream_t stream) {
    using namespace lsem;
    if (!args) return LSE_MERGE_ENULL;
    int64_t pitch = 0;
    int rc = noalloc_layout(args, &pitch);
    if (rc != LSE_MERGE_OK) return rc;
    if (args->rank_begin != 0 || args->rank_count != args->world) return LSE_MERGE_EDIMS;
    void* base = nullptr;
    const int se = noalloc_scratch(&base);
    if (se != 0) return fail_cuda(LSE_MERGE_ECUDA, se);
    lse_merge_cp_args a = *args;
    for (int q = 0; q < LSE_MERGE_CP_MAX_WORLD; ++q)
        a.ws[q] = q < a.world ? static_cast<char*>(base) + (int64_t)q * pitch : nullptr;
    // Validate before touching the array, so a rejected call changes nothing.
    rc = lse_merge_cp_validate(&a);
    if (rc != LSE_MERGE_OK) return rc;
    // Every call starts from zeroed headers: landed counters, status word,
    // completed-call count and finished-CTA count of each rank.
    const cudaError_t e = cudaMemset2DAsync(base, (size_t)pitch, 0, (size_t)kCpHeaderBytes,
                                            (size_t)a.world, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return lse_merge_cp_exchange_merge(&a, stream);
}

extern "C" int lse_merge_cp_noalloc_status(const lse_merge_cp_args* args, uint32_t* status) {
    using namespace lsem;
    if (!args || !status) return LSE_MERGE_ENULL;
    int64_t pitch = 0;
    const int rc = noalloc_layout(args, &pitch);
    if (rc != LSE_MERGE_OK) return rc;
    void* base = nullptr;
    const int se = noalloc_scratch(&base);
    if (se != 0) return fail_cuda(LSE_MERGE_ECUDA, se);
    // every call already enqueued on the device, on any stream, first
    cudaError_t e = cudaDeviceSynchronize();
    for (int q = 0; q < args->world && e == cudaSuccess; ++q)
        e = cudaMemcpy(status + q, static_cast<const char*>(base) + (int64_t)q * pitch +
                                       LSE_MERGE_CP_STATUS_OFFSET,
                       sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail_cuda(LSE_MERGE_ECUDA, (int)e);
    return LSE_MERGE_OK;
}
