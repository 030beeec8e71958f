// decode_attention.cu -- split-KV decode attention on sm_100a, optionally with
// the LSE-weighted merge of its partials fused in through a thread-block
// cluster.
//
// The producer of the merge's inputs (page "[flashinfer] FlashInfer의
// Context-Parallel Decode 최적화: Fused A2A + LSE Reduce", section "들어가며":
// each rank attends over its own KV shard and returns o_r and lse_r).  Here
// the shards are the R splits of one sequence's keys, computed by R CTAs.
//
// One CTA = one (batch b, KV head, split r), kAttnWarps warps.  The G query
// heads that share the KV head are the rows of a 16-row tile, so both
// products are tensor-core mma.sync m16n8k16 (bf16/fp16 in, fp32 accumulate):
//   S = Q K^T   A = Q (16 x D, registers), B = K^T from a shared-memory tile
//   O += P V    A = P (the S accumulators, exponentiated, as bf16/fp16),
//               B = V from a shared-memory tile (ldmatrix .trans)
// Each warp owns the key tiles w, w + kAttnWarps, ... of the split and a
// private ring of kAttnStages K/V tiles filled with cp.async (16-byte
// chunks, XOR-swizzled so ldmatrix rows hit distinct banks).  An online
// softmax (running max m and sum l in log2 units) keeps O unnormalised.
// After the key loop the warps' states are merged in shared memory (the
// LSE merge again, over the warps), giving the split's (o_r, lse_r).
//
//  * lse_merge_decode_partials writes (o_r, lse_r) to global memory.
//  * lse_merge_decode_attention_ws merges them in the same kernel without a
//    cluster: every split CTA writes its partial into the caller's
//    workspace, makes it visible device-wide and adds 1 to the (b, KV head)
//    counter there; the CTA that brings the counter to R merges the R
//    partials (read back through L2, where they still are), writes the
//    output and sets the counter back to 0 for the next call.  No CTA waits
//    for another; the partials never need to reach HBM before the merge.
//  * lse_merge_decode_attention launches the R splits of one (b, KV head) as
//    a cluster.  CTA r > 0 stores its split's partial into slot r of a
//    receive buffer in CTA 0's shared memory (distributed shared memory),
//    each thread then arrives, with release semantics at cluster scope, on
//    an mbarrier in CTA 0, and the CTA exits at once.  CTA 0 writes its own
//    partial into slot 0, waits on the mbarrier (bounded by the global
//    timer) and merges the R slots.  Only CTA 0 waits for the slowest split;
//    the others free their SM as soon as their keys are done.  The receive
//    buffer lies outside the K/V ring, which CTA 0 may still be using when a
//    sibling's partial arrives.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "lse_merge.h"
#include "plan.h"

namespace cg = cooperative_groups;

namespace lsem {
namespace attn {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Longest wait of CTA 0 for its siblings' partials (the siblings run at the
// same time as CTA 0, over as many keys, so the wait normally ends within a
// few microseconds).
constexpr uint64_t kFusedWaitNs = 2000000000ull;

struct AParams {
    const char* q;
    const char* k;
    const char* v;
    const int32_t* kv_len;
    int64_t q_b, q_h, k_b, k_h, k_l, v_b, v_h, v_l;   // BYTE strides
    int Hq, G, L, R;
    float scale_log2;      // scale * log2(e)
    float* po;             // partials [B, Hq, R, D] (unfused)
    float* pl;             // [B, Hq, R]
    char* out;             // merged output [B, Hq, D] (fused)
    float* out_lse;        // [B, Hq]
    unsigned* ws_cnt;      // workspace: arrived splits per (b, KV head) [B, Hkv]
    float* ws_l;           // workspace: split lse [B, Hkv, R, G]
    float* ws_o;           // workspace: split o [B, Hkv, R, G, D]
    int Hkv;
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// 16-byte global -> shared copy; `bytes` = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- cluster barrier and mbarrier (the fused merge's hand-off to CTA 0)
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Arrive on the mbarrier at shared address `bar` of cluster CTA `rank`, after
// (release, cluster scope) this thread's earlier stores.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar, uint32_t rank) {
    uint32_t rbar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(bar), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rbar) : "memory");
}
// One bounded probe of phase `parity` of the local mbarrier (acquire, cluster scope).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\n"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// Add v to *p (gpu scope, acquire and release); returns the old value.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
    __device__ static void run(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ static uint32_t pack(float lo, float hi) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};

template <>
struct Mma<__half> {
    __device__ static void run(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ static uint32_t pack(float lo, float hi) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};

template <typename TOut>
__device__ __forceinline__ void store_out(char* p, float x);
template <>
__device__ __forceinline__ void store_out<float>(char* p, float x) { *reinterpret_cast<float*>(p) = x; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(char* p, float x) {
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ void store_out<__half>(char* p, float x) {
    *reinterpret_cast<__half*>(p) = __float2half_rn(x);
}

// Shared-memory byte offset of 16-byte chunk `ch` of tile row `row` (rows of
// D*2 bytes): chunks are XOR-swizzled within groups of 8 so that the 8 rows
// one ldmatrix 8x8 matrix reads fall in 8 different bank groups.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int row, int ch) {
    return (uint32_t)(row * (D * 2) + ((ch ^ (row & 7)) * 16));
}

// What the kernel does with a split's partial (kAttnMode* of plan.h).
constexpr int kModePartials = kAttnModePartials;
constexpr int kModeCluster = kAttnModeCluster;
constexpr int kModeWorkspace = kAttnModeWorkspace;

// One work unit: split r of the keys of (batch b, KV head hk).  [lo, hi) are
// its keys; `mine` is how many of its key tiles the calling warp takes (the
// warps take tiles w, w + kAttnWarps, ...).
struct Unit {
    int b, hk, r, lo, hi, mine;
    const char* kb;   // K of (b, hk)
    const char* vb;   // V of (b, hk)
};

// Units are numbered with the split fastest, then the KV head, then the batch.
__device__ __forceinline__ Unit unit_of(const AParams& p, int r, int hk, int b, int warp) {
    constexpr int TK = kAttnTileKeys;
    Unit x;
    x.r = r;
    x.hk = hk;
    x.b = b;
    int len = p.L;
    if (p.kv_len) len = min(max(__ldg(p.kv_len + b), 0), p.L);
    const int per = (len + p.R - 1) / p.R;
    x.lo = min(len, r * per);
    x.hi = min(len, x.lo + per);
    const int ntiles = (x.hi - x.lo + TK - 1) / TK;
    x.mine = ntiles > warp ? (ntiles - warp + kAttnWarps - 1) / kAttnWarps : 0;
    x.kb = p.k + (int64_t)b * p.k_b + (int64_t)hk * p.k_h;
    x.vb = p.v + (int64_t)b * p.v_b + (int64_t)hk * p.v_h;
    return x;
}

// Q as the A operand of Q K^T: rows g and g+8 are query heads h0+g, h0+g+8
// (zero beyond the group), columns 16*ks + 2t (+1) and + 8.
template <int D>
__device__ __forceinline__ void load_q(const AParams& p, int b, int h0, int g, int t,
                                       uint32_t (&qa)[D / 16][4]) {
    const char* qb = p.q + (int64_t)b * p.q_b;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const int c0 = (ks * 16 + 2 * t) * 2;
        qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;
        if (g < p.G) {
            const char* row = qb + (int64_t)(h0 + g) * p.q_h;
            qa[ks][0] = __ldg(reinterpret_cast<const unsigned int*>(row + c0));
            qa[ks][2] = __ldg(reinterpret_cast<const unsigned int*>(row + c0 + 16));
        }
        if (g + 8 < p.G) {
            const char* row = qb + (int64_t)(h0 + g + 8) * p.q_h;
            qa[ks][1] = __ldg(reinterpret_cast<const unsigned int*>(row + c0));
            qa[ks][3] = __ldg(reinterpret_cast<const unsigned int*>(row + c0 + 16));
        }
    }
}

// Copy key tile `i` of the calling warp in unit `x` (keys lo + (warp +
// i*kAttnWarps)*TK ...) into the ring stage at shared address `kd` (K) and
// kd + TILE (V); keys at or past hi are zero-filled.
template <int D>
__device__ __forceinline__ void issue_tile(const AParams& p, const Unit& x, int warp, int i,
                                           uint32_t kd, int lane) {
    constexpr int TK = kAttnTileKeys;
    constexpr int CPR = D / 8;   // 16-byte chunks per K/V row
    constexpr int TILE = TK * D * 2;
    const int key0 = x.lo + (warp + i * kAttnWarps) * TK;
    const uint32_t vd = kd + TILE;
#pragma unroll 4
    for (int c = lane; c < TK * CPR; c += 32) {
        const int row = c / CPR, ch = c - row * CPR;
        const int key = key0 + row;
        const bool ok = key < x.hi;
        const int64_t src_key = ok ? key : x.lo;
        cp_async16(kd + tile_off<D>(row, ch), x.kb + src_key * p.k_l + ch * 16, ok ? 16 : 0);
        cp_async16(vd + tile_off<D>(row, ch), x.vb + src_key * p.v_l + ch * 16, ok ? 16 : 0);
    }
}

// The running state of a warp's online softmax over its key tiles: rows g
// and g+8 of the 16-row tile, in log2 units.
template <int D>
struct WarpState {
    float m0, m1;   // running max
    float l0, l1;   // this thread's share of the running sums
    float o[D / 8][4];
    __device__ __forceinline__ void reset() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    }
};

// Fold one K/V tile (K at shared address ks_u, V at ks_u + TILE; first key
// key0) into the warp's state: S = Q K^T, online softmax, O += P V.
template <typename T, int D>
__device__ __forceinline__ void attend_tile(uint32_t ks_u, const uint32_t (&qa)[D / 16][4],
                                            int key0, int hi, float scale_log2, int lane,
                                            WarpState<D>& w) {
    constexpr int TK = kAttnTileKeys;
    constexpr int KS = D / 16;   // k-steps of Q K^T
    constexpr int NT = D / 8;    // n-tiles of P V
    constexpr int TILE = TK * D * 2;
    constexpr int NJ = TK / 8;   // n-tiles of Q K^T (8 keys each)
    constexpr int KK = TK / 16;  // k-steps of P V (16 keys each)
    const uint32_t vs_u = ks_u + TILE;
    const int t = lane & 3;

    // ---- S = Q K^T: NJ n-tiles of 8 keys
    float sacc[NJ][4];
#pragma unroll
    for (int j = 0; j < NJ; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int jp = 0; jp < NJ / 2; ++jp) {
            const int mi = lane >> 3, rr = lane & 7;
            const int row = (2 * jp + (mi >> 1)) * 8 + rr;
            const int ch = 2 * ks + (mi & 1);
            uint32_t bf[4];
            ldsm_x4(ks_u + tile_off<D>(row, ch), bf);
            Mma<T>::run(sacc[2 * jp], qa[ks], bf[0], bf[1]);
            Mma<T>::run(sacc[2 * jp + 1], qa[ks], bf[2], bf[3]);
        }
    }

    // ---- online softmax over this tile (scores in log2 units)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool ok = key0 + 8 * j + 2 * t + e < hi;
            sacc[j][e] = ok ? sacc[j][e] * scale_log2 : -INFINITY;
            sacc[j][e + 2] = ok ? sacc[j][e + 2] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sacc[j][e]);
            mx1 = fmaxf(mx1, sacc[j][e + 2]);
        }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
    // every tile holds at least one valid key, so the new maxima are finite
    const float n0 = fmaxf(w.m0, mx0), n1 = fmaxf(w.m1, mx1);
    const float a0 = exp2f(w.m0 - n0), a1 = exp2f(w.m1 - n1);   // 0 on the first tile
    w.m0 = n0;
    w.m1 = n1;
    w.l0 *= a0;
    w.l1 *= a1;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        w.o[n][0] *= a0;
        w.o[n][1] *= a0;
        w.o[n][2] *= a1;
        w.o[n][3] *= a1;
    }
    uint32_t pa[KK][4];   // P as the A operand of the 16-key k-steps
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const float p0 = exp2f(sacc[j][0] - n0), p1 = exp2f(sacc[j][1] - n0);
        const float p2 = exp2f(sacc[j][2] - n1), p3 = exp2f(sacc[j][3] - n1);
        w.l0 += p0 + p1;
        w.l1 += p2 + p3;
        pa[j >> 1][(j & 1) * 2 + 0] = Mma<T>::pack(p0, p1);
        pa[j >> 1][(j & 1) * 2 + 1] = Mma<T>::pack(p2, p3);
    }

    // ---- O += P V: D/8 n-tiles, KK k-steps of 16 keys
#pragma unroll
    for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            const int mi = lane >> 3, rr = lane & 7;
            const int row = 16 * kk + (mi & 1) * 8 + rr;
            const int ch = 2 * np + (mi >> 1);
            uint32_t bf[4];
            ldsm_x4_t(vs_u + tile_off<D>(row, ch), bf);
            Mma<T>::run(w.o[2 * np], pa[kk], bf[0], bf[1]);
            Mma<T>::run(w.o[2 * np + 1], pa[kk], bf[2], bf[3]);
        }
    }
}

// Run the calling warp's share of unit `x`: its ring (shared address ring_u,
// kAttnStages stages) already holds, or is being filled with, its first
// kAttnStages - 1 tiles (one cp.async group each).  On return every copy of
// the ring has landed and been read, and w holds the warp's state with the
// sums l0, l1 complete over the quad.
template <typename T, int D>
__device__ __forceinline__ void attend_unit(const AParams& p, const Unit& x, int warp, int lane,
                                            uint32_t ring_u, const uint32_t (&qa)[D / 16][4],
                                            WarpState<D>& w) {
    constexpr int TK = kAttnTileKeys;
    constexpr int S = kAttnStages;
    constexpr int TILE = TK * D * 2;
    w.reset();
    for (int i = 0; i < x.mine; ++i) {
        if (i + S - 1 < x.mine)
            issue_tile<D>(p, x, warp, i + S - 1, ring_u + (uint32_t)(((i + S - 1) % S) * 2 * TILE), lane);
        cp_commit();
        cp_wait<S - 1>();
        __syncwarp();
        const int key0 = x.lo + (warp + i * kAttnWarps) * TK;
        attend_tile<T, D>(ring_u + (uint32_t)((i % S) * 2 * TILE), qa, key0, x.hi, p.scale_log2, lane, w);
        __syncwarp();
    }
    cp_wait<0>();
    __syncwarp();
    w.l0 += __shfl_xor_sync(kFull, w.l0, 1);
    w.l0 += __shfl_xor_sync(kFull, w.l0, 2);
    w.l1 += __shfl_xor_sync(kFull, w.l1, 1);
    w.l1 += __shfl_xor_sync(kFull, w.l1, 2);
}

// Issue the first kAttnStages - 1 tiles of the calling warp's share of unit
// x into its ring, one cp.async group per stage (empty groups past `mine`).
template <int D>
__device__ __forceinline__ void issue_prologue(const AParams& p, const Unit& x, int warp, int lane,
                                               uint32_t ring_u) {
    constexpr int S = kAttnStages;
    constexpr int TILE = kAttnTileKeys * D * 2;
#pragma unroll
    for (int s = 0; s < S - 1; ++s) {
        if (s < x.mine) issue_tile<D>(p, x, warp, s, ring_u + (uint32_t)(s * 2 * TILE), lane);
        cp_commit();
    }
}

// Warp states in shared memory for the merge over the warps, G rows per
// warp: m [kAttnWarps*G], l [kAttnWarps*G], o [kAttnWarps*G][D] (fp32).
template <int D>
__device__ __forceinline__ void store_warp_state(float* st, int G, int warp, int lane,
                                                 const WarpState<D>& w) {
    const int g = lane >> 2, t = lane & 3;
    float* st_m = st;
    float* st_l = st_m + kAttnWarps * G;
    float* st_o = st_l + kAttnWarps * G;
    if (t == 0) {
        if (g < G) {
            st_m[warp * G + g] = w.m0;
            st_l[warp * G + g] = w.l0;
        }
        if (g + 8 < G) {
            st_m[warp * G + g + 8] = w.m1;
            st_l[warp * G + g + 8] = w.l1;
        }
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        if (g < G) {
            float* o0 = st_o + (warp * G + g) * D + 8 * n + 2 * t;
            o0[0] = w.o[n][0];
            o0[1] = w.o[n][1];
        }
        if (g + 8 < G) {
            float* o1 = st_o + (warp * G + g + 8) * D + 8 * n + 2 * t;
            o1[0] = w.o[n][2];
            o1[1] = w.o[n][3];
        }
    }
}

// The split's (o, lse) of element (gg, d): the LSE merge of the warps'
// states (lse in natural-log units; an empty split gives 0 and -inf).
template <int D>
__device__ __forceinline__ void merge_warp_states(const float* st, int G, int gg, int d, float& o,
                                                  float& lse) {
    const float* st_m = st;
    const float* st_l = st_m + kAttnWarps * G;
    const float* st_o = st_l + kAttnWarps * G;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, st_m[w * G + gg]);
    float den = 0.f, num = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float mw = st_m[w * G + gg];
            if (mw != -INFINITY) {
                const float e = exp2f(mw - M);
                den += e * st_l[w * G + gg];
                num += e * st_o[(w * G + gg) * D + d];
            }
        }
    }
    o = den > 0.f ? num / den : 0.f;
    lse = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
}

// Workspace form, in the CTA that brought the (b, KV head) counter to R:
// merge the R split partials of the group (ws_o [R][G][D], ws_l [R][G],
// written moments ago, so read through L2) into the output rows
// rows_b .. rows_b + G - 1.  Each thread takes up to kMergeOut output
// elements and walks the splits in batches of kMergeBatch, the lse and o
// loads of a whole batch issued before any is used, then folded into a
// running (max, weight sum, weighted sum) per element -- one L2 round trip
// per batch, none for the weights alone.  An empty split has lse -inf, o 0.
template <typename TOut, int D>
__device__ __forceinline__ void merge_workspace(const AParams& p, const float* ws_o,
                                                const float* ws_l, int64_t rows_b, int tid,
                                                int nthr) {
    constexpr int kMergeBatch = 4, kMergeOut = 4;
    const int G = p.G, R = p.R;
    const int GD = G * D;
    for (int base = tid; base < GD; base += kMergeOut * nthr) {
        float mx[kMergeOut], den[kMergeOut], num[kMergeOut];
#pragma unroll
        for (int k = 0; k < kMergeOut; ++k) {
            mx[k] = -INFINITY;
            den[k] = num[k] = 0.f;
        }
        for (int j0 = 0; j0 < R; j0 += kMergeBatch) {
            float lv[kMergeOut][kMergeBatch], ov[kMergeOut][kMergeBatch];
#pragma unroll
            for (int k = 0; k < kMergeOut; ++k) {
                const int idx = base + k * nthr;
                const int gg = idx < GD ? idx / D : 0, d = idx - gg * D;
#pragma unroll
                for (int u = 0; u < kMergeBatch; ++u) {
                    const int j = j0 + u;
                    const bool in = idx < GD && j < R;
                    lv[k][u] = in ? __ldcg(ws_l + j * G + gg) : -INFINITY;
                    ov[k][u] = in ? __ldcg(ws_o + ((int64_t)j * G + gg) * D + d) : 0.f;
                }
            }
#pragma unroll
            for (int k = 0; k < kMergeOut; ++k) {
                float bm = mx[k];
#pragma unroll
                for (int u = 0; u < kMergeBatch; ++u) bm = fmaxf(bm, lv[k][u]);
                const float ref = bm == -INFINITY ? 0.f : bm;
                const float sc = expf(mx[k] - ref);   // 0 while nothing was seen
                den[k] *= sc;
                num[k] *= sc;
#pragma unroll
                for (int u = 0; u < kMergeBatch; ++u) {
                    const float e = expf(lv[k][u] - ref);   // 0 for an empty split
                    den[k] += e;
                    num[k] = fmaf(e, ov[k][u], num[k]);
                }
                mx[k] = bm;
            }
        }
#pragma unroll
        for (int k = 0; k < kMergeOut; ++k) {
            const int idx = base + k * nthr;
            if (idx < GD) {
                const int gg = idx / D, d = idx - gg * D;
                const int64_t row = rows_b + gg;
                store_out<TOut>(p.out + (row * D + d) * (int64_t)sizeof(TOut),
                                den[k] > 0.f ? num[k] / den[k] : 0.f);
                if (d == 0) p.out_lse[row] = den[k] > 0.f ? mx[k] + logf(den[k]) : -INFINITY;
            }
        }
    }
}

// One CTA per unit (grid R x Hkv x B); the cluster form needs this shape
// (the R splits of a (b, KV head) are one cluster along x).
template <typename T, int D, int MODE, typename TOut>
__global__ void __launch_bounds__(kAttnWarps * 32, 1) decode_attn_kernel(const AParams p) {
    constexpr int TILE = kAttnTileKeys * D * 2;
    extern __shared__ __align__(128) unsigned char smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int r = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int G = p.G, R = p.R;
    const int h0 = hk * G;

    // Cluster: CTA 0's receive buffer behind the ring and the warp states:
    // the mbarrier (16 bytes), lse [R][G], then o [R][G][D] (fp32).  r is
    // the CTA's rank in its cluster (the cluster spans the R splits along x).
    constexpr int64_t kRing = (int64_t)kAttnWarps * kAttnStages * 2 * TILE;
    constexpr int64_t kStates = (int64_t)kAttnWarps * 16 * (D + 2) * 4;
    constexpr int64_t kRecvOff = ((kRing > kStates ? kRing : kStates) + 15) / 16 * 16;
    const uint32_t bar = smem_u32(smem + kRecvOff);
    float* const recv_l = reinterpret_cast<float*>(smem + kRecvOff + 16);
    float* const recv_o = recv_l + ((R * G + 3) & ~3);
    if constexpr (MODE == kModeCluster) {
        if (R > 1) {
            if (r == 0 && threadIdx.x == 0) mbar_init(bar, (uint32_t)((R - 1) * blockDim.x));
            // the barrier's init is visible to every CTA before any arrives on
            // it: each thread waits on this cluster barrier before its first
            // store into CTA 0
            cluster_arrive_release();
        }
    }

    pdl_wait();
    pdl_release();

    const Unit x = unit_of(p, r, hk, b, warp);
    const uint32_t ring_u = smem_u32(smem + (size_t)warp * kAttnStages * 2 * TILE);
    uint32_t qa[D / 16][4];
    load_q<D>(p, b, h0, g, t, qa);
    issue_prologue<D>(p, x, warp, lane, ring_u);
    WarpState<D> w;
    attend_unit<T, D>(p, x, warp, lane, ring_u, qa, w);
    __syncthreads();   // every warp is done with its ring: reuse the shared memory

    // ---- merge the warps' states
    float* st = reinterpret_cast<float*>(smem);
    store_warp_state<D>(st, G, warp, lane, w);
    __syncthreads();
    const int64_t rows_b = (int64_t)b * p.Hq + h0;
    // Cluster: this split's partial goes to slot r of CTA 0's receive buffer.
    // Workspace: to slot r of this (b, KV head)'s block of the workspace.
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    float* dst_o = recv_o;
    float* dst_l = recv_l;
    if constexpr (MODE == kModeWorkspace) {
        dst_o = p.ws_o + bh * R * G * D;
        dst_l = p.ws_l + bh * R * G;
    }
    if constexpr (MODE == kModeCluster) {
        if (R > 1) {
            cluster_wait_acquire();   // CTA 0's mbarrier is initialised
            if (r != 0) {
                cg::cluster_group cluster = cg::this_cluster();
                dst_o = cluster.map_shared_rank(recv_o, 0);
                dst_l = cluster.map_shared_rank(recv_l, 0);
            }
        }
    }
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int gg = idx / D, d = idx - gg * D;
        float o, lse;
        merge_warp_states<D>(st, G, gg, d, o, lse);
        if constexpr (MODE != kModePartials) {
            dst_o[(r * G + gg) * D + d] = o;
            if (d == 0) dst_l[r * G + gg] = lse;
        } else {
            const int64_t row = rows_b + gg;
            p.po[(row * R + r) * D + d] = o;
            if (d == 0) p.pl[row * R + r] = lse;
        }
    }

    if constexpr (MODE == kModeWorkspace) {
        // ---- count this split in; the last of the R splits merges them all.
        // The CTA barrier orders every thread's partial stores before thread
        // 0's count, whose release (gpu scope, cumulative) publishes them;
        // the count's acquire makes the splits counted before visible to the
        // last CTA, whose threads read them after the second barrier.
        __shared__ int s_last;
        __syncthreads();
        if (threadIdx.x == 0) s_last = atom_add_acq_rel_gpu(p.ws_cnt + bh, 1u) == (unsigned)(R - 1);
        __syncthreads();
        if (!s_last) return;
        merge_workspace<TOut, D>(p, dst_o, dst_l, rows_b, threadIdx.x, blockDim.x);
        if (threadIdx.x == 0) p.ws_cnt[bh] = 0u;   // every split of this call has counted
    }
    if constexpr (MODE == kModeCluster) {
        // ---- hand the partial to CTA 0, which merges the R splits
        if (R > 1 && r != 0) {
            mbar_arrive_remote(bar, 0);   // after this thread's stores into CTA 0
            return;                       // nothing reads this CTA's shared memory
        }
        bool ok = true;
        if (R > 1) {
            // every sibling thread arrives once: phase 0 completes when all
            // R - 1 partials are in recv; bounded wait (a sibling that never
            // arrives would be a bug: the result is then NaN, not a hang)
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(bar, 0)) {
                if (global_ns() - t0 > kFusedWaitNs) {
                    ok = false;
                    break;
                }
            }
        }
        ok = __syncthreads_and(ok) != 0;   // also orders CTA 0's own slot-0 stores
        for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
            const int gg = idx / D, d = idx - gg * D;
            float M = -INFINITY;
            for (int j = 0; j < R; ++j) M = fmaxf(M, recv_l[j * G + gg]);
            float den = 0.f, num = 0.f;
            if (M != -INFINITY) {
                for (int j = 0; j < R; ++j) {
                    const float lj = recv_l[j * G + gg];
                    if (lj != -INFINITY) {   // an empty split's o is not used
                        const float e = expf(lj - M);
                        den += e;
                        num += e * recv_o[(j * G + gg) * D + d];
                    }
                }
            }
            const int64_t row = rows_b + gg;
            float o = den > 0.f ? num / den : 0.f;
            float lse = den > 0.f ? M + logf(den) : -INFINITY;
            if (!ok) o = lse = __int_as_float(0x7fc00000);   // NaN: the hand-off never completed
            store_out<TOut>(p.out + (row * D + d) * (int64_t)sizeof(TOut), o);
            if (d == 0) p.out_lse[row] = lse;
        }
    }
}

using AttnFn = void (*)(AParams);

template <typename T, int D, int MODE>
AttnFn pick_o(int out_dtype) {
    switch (out_dtype) {
        case LSE_MERGE_F32: return decode_attn_kernel<T, D, MODE, float>;
        case LSE_MERGE_F16: return decode_attn_kernel<T, D, MODE, __half>;
        default: return decode_attn_kernel<T, D, MODE, __nv_bfloat16>;
    }
}
template <typename T, int D>
AttnFn pick_d(int mode, int out_dtype) {
    if (mode == kModePartials) return decode_attn_kernel<T, D, kModePartials, float>;
    return mode == kModeCluster ? pick_o<T, D, kModeCluster>(out_dtype)
                                : pick_o<T, D, kModeWorkspace>(out_dtype);
}
template <typename T>
AttnFn pick_t(int D, int mode, int out_dtype) {
    return D == 64 ? pick_d<T, 64>(mode, out_dtype) : pick_d<T, 128>(mode, out_dtype);
}
AttnFn pick(int dtype, int D, int mode, int out_dtype) {
    return dtype == LSE_MERGE_F16 ? pick_t<__half>(D, mode, out_dtype)
                                  : pick_t<__nv_bfloat16>(D, mode, out_dtype);
}

// cudaFuncSetAttribute per (kernel, device) for dynamic shared memory above
// 48 KB, raised whenever a launch needs more than the size set so far (the
// fused kernel's receive buffer grows with R and the group size).
std::mutex g_attr_mu;
struct AttrDone {
    const void* fn;
    int dev;
    int64_t bytes;
};
AttrDone g_attr_done[128];
int g_attr_n = 0;

cudaError_t ensure_smem(AttnFn fn, int64_t bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_attr_mu);
    AttrDone* slot = nullptr;
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr_done[i].fn == (const void*)fn && g_attr_done[i].dev == dev) slot = &g_attr_done[i];
    if (slot && slot->bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    if (slot)
        slot->bytes = bytes;
    else if (g_attr_n < 128)
        g_attr_done[g_attr_n++] = AttrDone{(const void*)fn, dev, bytes};
    return cudaSuccess;
}

int launch(const void* q, const void* k, const void* v, const int32_t* kv_len, int B, int Hq,
           int Hkv, int L, int D, int R, float scale, const lse_merge_attn_strides* strides,
           int dtype, int out_dtype, void* out_o, float* out_lse, int mode, void* ws,
           int64_t ws_bytes, cudaStream_t stream) {
    if (Hq < 1 || Hkv < 1 || L < 1 || D < 1) return LSE_MERGE_EDIMS;
    const lse_merge_attn_strides st = strides ? *strides : default_attn_strides(Hq, Hkv, L, D);
    const bool fused = mode != kModePartials;
    AttnPlan pl;
    const int rc = make_attn_plan(q, k, v, B, Hq, Hkv, L, D, R, scale, st, dtype,
                                  fused ? out_dtype : LSE_MERGE_F32, out_o, out_lse, mode, ws,
                                  ws_bytes, &pl);
    if (rc != LSE_MERGE_OK) return rc;
    AParams ap{};
    ap.q = static_cast<const char*>(q);
    ap.k = static_cast<const char*>(k);
    ap.v = static_cast<const char*>(v);
    ap.kv_len = kv_len;
    ap.q_b = st.q_b * 2;
    ap.q_h = st.q_h * 2;
    ap.k_b = st.k_b * 2;
    ap.k_h = st.k_h * 2;
    ap.k_l = st.k_l * 2;
    ap.v_b = st.v_b * 2;
    ap.v_h = st.v_h * 2;
    ap.v_l = st.v_l * 2;
    ap.Hq = Hq;
    ap.Hkv = Hkv;
    ap.G = pl.G;
    ap.L = L;
    ap.R = R;
    ap.scale_log2 = scale * kLog2e;
    ap.po = fused ? nullptr : static_cast<float*>(out_o);
    ap.pl = fused ? nullptr : out_lse;
    ap.out = fused ? static_cast<char*>(out_o) : nullptr;
    ap.out_lse = fused ? out_lse : nullptr;
    if (mode == kModeWorkspace) {
        char* w = static_cast<char*>(ws);
        ap.ws_cnt = reinterpret_cast<unsigned*>(w);
        ap.ws_l = reinterpret_cast<float*>(w + pl.ws_l_off);
        ap.ws_o = reinterpret_cast<float*>(w + pl.ws_o_off);
    }
    const AttnFn fn = pick(dtype, D, mode, out_dtype);
    cudaError_t e = ensure_smem(fn, pl.smem);
    if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)R, (unsigned)Hkv, (unsigned)B);
        cfg.blockDim = dim3(kAttnWarps * 32);
        cfg.dynamicSmemBytes = (size_t)pl.smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (kPdl) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        if (mode == kModeCluster) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = (unsigned)R;
            attr[na].val.clusterDim.y = 1;
            attr[na].val.clusterDim.z = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        e = cudaLaunchKernelEx(&cfg, fn, ap);
    }
    if (e != cudaSuccess) {
        set_last_cuda_error((int)e);
        (void)cudaGetLastError();
        return LSE_MERGE_ELAUNCH;
    }
    return LSE_MERGE_OK;
}

}  // namespace
}  // namespace attn
}  // namespace lsem

extern "C" {

int lse_merge_decode_partials(const void* q, const void* k, const void* v, const int32_t* kv_len,
                              int B, int Hq, int Hkv, int L, int D, int R, float scale,
                              const lse_merge_attn_strides* strides, int dtype,
                              float* partial_o, float* partial_lse, lse_merge_stream_t stream) {
    return lsem::attn::launch(q, k, v, kv_len, B, Hq, Hkv, L, D, R, scale, strides, dtype,
                              LSE_MERGE_F32, partial_o, partial_lse, lsem::kAttnModePartials,
                              nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

int lse_merge_decode_attention(const void* q, const void* k, const void* v, const int32_t* kv_len,
                               int B, int Hq, int Hkv, int L, int D, int R, float scale,
                               const lse_merge_attn_strides* strides, int dtype, int out_dtype,
                               void* out_o, float* out_lse, lse_merge_stream_t stream) {
    return lsem::attn::launch(q, k, v, kv_len, B, Hq, Hkv, L, D, R, scale, strides, dtype,
                              out_dtype, out_o, out_lse, lsem::kAttnModeCluster, nullptr, 0,
                              reinterpret_cast<cudaStream_t>(stream));
}

int lse_merge_decode_attention_ws(const void* q, const void* k, const void* v,
                                  const int32_t* kv_len, int B, int Hq, int Hkv, int L, int D,
                                  int R, float scale, const lse_merge_attn_strides* strides,
                                  int dtype, int out_dtype, void* workspace,
                                  int64_t workspace_bytes, void* out_o, float* out_lse,
                                  lse_merge_stream_t stream) {
    return lsem::attn::launch(q, k, v, kv_len, B, Hq, Hkv, L, D, R, scale, strides, dtype,
                              out_dtype, out_o, out_lse, lsem::kAttnModeWorkspace, workspace,
                              workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
