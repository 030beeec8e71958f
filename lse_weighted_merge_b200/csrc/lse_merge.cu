// lse_merge.cu -- sm_100a kernels and the C entry points of the LSE-weighted merge.
//
// The operation (page "[flashinfer] FlashInfer의 Context-Parallel Decode 최적화:
// Fused A2A + LSE Reduce", section "코드 분석 / 1. Fused Kernel 구현": weights
// from the lse values, fp32 accumulation over the partial axis, division by
// the sum of the weights, conversion to FP16/BF16; the KV-shard partials
// o_r, lse_r are introduced in section "들어가며"):
//     m = max_r lse_r,  e_r = exp(lse_r - m),  out = sum_r e_r o_r / sum_r e_r,
//     out_lse = m + log(sum_r e_r);   all shards empty -> out = 0, out_lse = -inf.
//
// The merge moves R*D input elements per (b,h) row for 2 flops each, so it is
// bound by HBM bandwidth and uses no tensor cores.  Design:
//   * a row (or a slice of a long row) belongs to a group of `lanes`
//     consecutive lanes of one warp; each lane owns 16 contiguous bytes of
//     every partial row (8 bf16/fp16 or 4 fp32 elements);
//   * each lane issues the 16-byte loads of RC partial rows before it needs
//     any weight, so RC * 16 bytes per lane are in flight while the lse
//     values are still being reduced;
//   * lane j of a group holds lse_j; max and sum are group shuffles, and
//     the weight of partial i is broadcast from lane i by a shuffle;
//   * accumulation in fp32 registers, one reciprocal of the weight sum,
//     round-to-nearest-even conversion, 16-byte stores;
//   * a partial with weight 0 is skipped by a select, so NaN stored in an
//     empty shard cannot reach the output.
// The partial rows are streamed once: loads bypass L1 and ask L2 for 256-byte
// prefetch (the neighbouring lanes' sectors of the same row).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "device_common.cuh"
#include "lse_merge.h"
#include "plan.h"

namespace lsem {
namespace {

constexpr unsigned kFull = 0xffffffffu;

struct KParams {
    const char* o;      // partial_o
    const float* lse;   // partial_lse
    char* out;          // out_o, dense [B,H,D]
    float* out_lse;     // dense [B,H]
    int64_t o_r, o_b, o_h;  // partial_o strides in BYTES
    int64_t l_r, l_b, l_h;  // partial_lse strides in elements
    int R, H, D;
    int dv;             // 16-byte vectors per row (vector kernels)
    int lanes, lg;      // lanes per group, log2(lanes)
    int spr;            // groups (slices) per row
    int64_t groups;     // total groups
    // n / spr and n / H for 32-bit n by one high multiply (d == 1: n itself);
    // used when every group and row index fits in 32 bits (idx32).
    uint64_t c_spr, c_H;
    int idx32;
};

// Row, slice, batch and head of group `grp` (valid when grp < groups).
struct RowIdx {
    int64_t row, b, h;
    int slice;
};
__device__ __forceinline__ RowIdx row_of(const KParams& p, int64_t grp) {
    RowIdx r;
    if (p.idx32) {
        const uint32_t g = (uint32_t)grp;
        const uint32_t q = fastdiv(g, p.c_spr, (uint32_t)p.spr);
        const uint32_t bb = fastdiv(q, p.c_H, (uint32_t)p.H);
        r.row = q;
        r.slice = (int)(g - q * (uint32_t)p.spr);
        r.b = bb;
        r.h = q - bb * (uint32_t)p.H;
    } else {
        r.row = grp / p.spr;
        r.slice = (int)(grp - r.row * p.spr);
        r.b = r.row / p.H;
        r.h = r.row - r.b * p.H;
    }
    return r;
}

// --------------------------------------------------------------- group reductions

// Groups are `lanes` consecutive lanes starting at a multiple of `lanes`, so an
// xor offset below `lanes` stays inside the group.
__device__ __forceinline__ float group_max(float v, int lanes) {
    for (int off = lanes >> 1; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
    return v;
}

__device__ __forceinline__ float group_sum(float v, int lanes) {
    for (int off = lanes >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    return v;
}

// ------------------------------------------------------------------ vector kernel

// Fold partial x (NV 16-byte columns) with weight w into acc.
template <typename TIn, int NV, int N2>
__device__ __forceinline__ void fold(uint64_t (&acc)[NV][N2], const uint4 (&x)[NV], float w) {
    const uint64_t ww = pack2f(w, w);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        uint64_t xx[N2];
        Elem<TIn>::unpack2(x[k], xx);
#pragma unroll
        for (int q = 0; q < N2; ++q) fma2(acc[k][q], xx[q], ww);
    }
}

// Scale acc by inv and store the NV columns of this lane (those inside the row).
template <typename TOut, int NV, int N, int N2>
__device__ __forceinline__ void store_cols(const KParams& p, int64_t row, int v0, bool live,
                                           const uint64_t (&acc)[NV][N2], float inv) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int v = v0 + k * p.lanes;
        if (live && v < p.dv) {
            float f[N];
#pragma unroll
            for (int q = 0; q < N2; ++q) {
                unpack2f(acc[k][q], f[2 * q], f[2 * q + 1]);
                f[2 * q] *= inv;
                f[2 * q + 1] *= inv;
            }
            store_vec<TOut, N>(p.out + (row * p.D + (int64_t)v * N) * (int64_t)sizeof(TOut), f);
        }
    }
}

// One group of p.lanes lanes merges one slice of one (b,h) row.  Lane j owns
// the 16-byte column v = slice*lanes + j of every partial row.  Control flow
// that reaches a shuffle depends only on R, lanes and RC, which are the same
// for every thread of the grid, so every shuffle sees all 32 lanes.
// This is the form with one 16-byte column per lane (NV = 1), used whenever
// the planner gives a lane a single column.
template <typename TIn, typename TOut, int RC>
__global__ void __launch_bounds__(kBlock, kMinBlocksVec1) merge_vec1_kernel(const KParams p) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t grp = t >> p.lg;
    const int j = (int)(t & (p.lanes - 1));
    const bool live = grp < p.groups;
    const RowIdx ri = row_of(p, live ? grp : 0);
    const int v = ri.slice * p.lanes + j;
    const bool vlive = live && v < p.dv;
    const char* orow = p.o + ri.b * p.o_b + ri.h * p.o_h + (int64_t)v * 16;
    const float* lrow = p.lse + ri.b * p.l_b + ri.h * p.l_h;
    if (kPrefetch) {   // the first RC partial rows, while the previous grid drains
#pragma unroll
        for (int i = 0; i < RC; ++i)
            if (vlive && i < p.R) prefetch_l2(orow + (int64_t)i * p.o_r);
        if (live && j < p.R) prefetch_l2(lrow + (int64_t)j * p.l_r);
    }
    pdl_wait();
    pdl_release();

    // Partial rows 0..RC-1 go in flight first; nothing here waits on lse.
    uint4 x[RC];
#pragma unroll
    for (int i = 0; i < RC; ++i) {
        x[i] = make_uint4(0u, 0u, 0u, 0u);
        if (vlive && i < p.R) x[i] = ld_stream16(orow + (int64_t)i * p.o_r);
    }

    // m = max_r lse_r over the group (lane j reads lse_j, lse_{j+lanes}, ...).
    float l0 = -INFINITY;
    if (live && j < p.R) l0 = __ldg(lrow + (int64_t)j * p.l_r);
    float m = l0;
    for (int c = p.lanes; c < p.R; c += p.lanes)
        if (live && c + j < p.R) m = fmaxf(m, __ldg(lrow + (int64_t)(c + j) * p.l_r));
    m = group_max(m, p.lanes);
    // An all-empty row has m = -inf; subtracting 0 instead keeps every weight
    // exp(-inf) = 0 rather than exp(-inf + inf) = NaN.
    const float mref = (m == -INFINITY) ? 0.f : m;

    uint64_t acc[N2];
#pragma unroll
    for (int k = 0; k < N2; ++k) acc[k] = 0ull;
    float esum = 0.f;

    for (int c = 0; c < p.R; c += p.lanes) {
        float l = l0;
        if (c > 0) {
            l = -INFINITY;
            if (live && c + j < p.R) l = __ldg(lrow + (int64_t)(c + j) * p.l_r);
        }
        const float e = expf(l - mref);  // weight of partial c+j; 0 for an empty shard
        esum += e;
        const int cn = min(p.R - c, p.lanes);
        // Warp-uniform: does any group of this warp have a zero weight in this
        // chunk?  Only then is the per-partial test needed (a partial of weight
        // 0 may hold NaN and must not reach the sum).
        const bool any_zero = __any_sync(kFull, j < cn && e == 0.f);
        for (int s0 = 0; s0 < cn; s0 += RC) {
            if (c > 0 || s0 > 0) {
#pragma unroll
                for (int i = 0; i < RC; ++i)
                    if (vlive && s0 + i < cn) x[i] = ld_stream16(orow + (int64_t)(c + s0 + i) * p.o_r);
            }
            auto fold_chunk = [&](auto check) {
#pragma unroll
                for (int i = 0; i < RC; ++i) {
                    const float w = __shfl_sync(kFull, e, s0 + i, p.lanes);
                    if (s0 + i < cn && (!decltype(check)::value || w != 0.f)) {
                        uint64_t xx[N2];
                        Elem<TIn>::unpack2(x[i], xx);
                        const uint64_t ww = pack2f(w, w);
#pragma unroll
                        for (int k = 0; k < N2; ++k) fma2(acc[k], xx[k], ww);
                    }
                }
            };
            if (any_zero) fold_chunk(std::true_type{});
            else fold_chunk(std::false_type{});
        }
    }
    esum = group_sum(esum, p.lanes);

    // esum >= 1 for a row with a finite max (its own weight is exp(0)).
    const float inv = esum > 0.f ? 1.f / esum : 0.f;
    if (vlive) {
        float f[N];
#pragma unroll
        for (int k = 0; k < N2; ++k) {
            unpack2f(acc[k], f[2 * k], f[2 * k + 1]);
            f[2 * k] *= inv;
            f[2 * k + 1] *= inv;
        }
        store_vec<TOut, N>(p.out + (ri.row * p.D + (int64_t)v * N) * (int64_t)sizeof(TOut), f);
    }
    if (live && ri.slice == 0 && j == 0) p.out_lse[ri.row] = esum > 0.f ? m + logf(esum) : -INFINITY;
}


// One group of p.lanes lanes merges one slice of one (b,h) row.  Lane j owns
// the NV 16-byte columns v0 + k*lanes (v0 = slice*lanes*NV + j, k < NV) of
// every partial row, so each warp load instruction reads lanes*16 contiguous
// bytes of a partial row.  Control flow that reaches a shuffle depends only
// on R, lanes, RC and NV, which are the same for every thread of the grid,
// so every shuffle sees all 32 lanes.
template <typename TIn, typename TOut, int RC, int NV>
__global__ void __launch_bounds__(kBlock, kMinBlocks) merge_vec_kernel(const KParams p) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t grp = t >> p.lg;
    const int j = (int)(t & (p.lanes - 1));
    const bool live = grp < p.groups;
    const RowIdx ri = row_of(p, live ? grp : 0);
    const int v0 = ri.slice * p.lanes * NV + j;
    const char* orow = p.o + ri.b * p.o_b + ri.h * p.o_h + (int64_t)v0 * 16;
    const float* lrow = p.lse + ri.b * p.l_b + ri.h * p.l_h;
    bool cl[NV];   // column k of this lane lies inside the row
#pragma unroll
    for (int k = 0; k < NV; ++k) cl[k] = live && v0 + k * p.lanes < p.dv;
    if (kPrefetch) {   // the first RC partial rows, while the previous grid drains
#pragma unroll
        for (int i = 0; i < RC; ++i)
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (cl[k] && i < p.R) prefetch_l2(orow + (int64_t)i * p.o_r + k * p.lanes * 16);
        if (live && j < p.R) prefetch_l2(lrow + (int64_t)j * p.l_r);
    }
    pdl_wait();
    pdl_release();

    // Partial rows 0..RC-1 go in flight first; nothing here waits on lse.
    uint4 x[RC][NV];
#pragma unroll
    for (int i = 0; i < RC; ++i)
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            x[i][k] = make_uint4(0u, 0u, 0u, 0u);
            if (cl[k] && i < p.R) x[i][k] = ld_stream16(orow + (int64_t)i * p.o_r + k * p.lanes * 16);
        }

    // m = max_r lse_r over the group (lane j reads lse_j, lse_{j+lanes}, ...).
    float l0 = -INFINITY;
    if (live && j < p.R) l0 = __ldg(lrow + (int64_t)j * p.l_r);
    float m = l0;
    for (int c = p.lanes; c < p.R; c += p.lanes)
        if (live && c + j < p.R) m = fmaxf(m, __ldg(lrow + (int64_t)(c + j) * p.l_r));
    m = group_max(m, p.lanes);
    // An all-empty row has m = -inf; subtracting 0 instead keeps every weight
    // exp(-inf) = 0 rather than exp(-inf + inf) = NaN.
    const float mref = (m == -INFINITY) ? 0.f : m;

    uint64_t acc[NV][N2];
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int q = 0; q < N2; ++q) acc[k][q] = 0ull;
    float esum = 0.f;

    for (int c = 0; c < p.R; c += p.lanes) {
        float l = l0;
        if (c > 0) {
            l = -INFINITY;
            if (live && c + j < p.R) l = __ldg(lrow + (int64_t)(c + j) * p.l_r);
        }
        const float e = expf(l - mref);  // weight of partial c+j; 0 for an empty shard
        esum += e;
        const int cn = min(p.R - c, p.lanes);
        // Warp-uniform: does any group of this warp have a zero weight in this
        // chunk?  Only then is the per-partial test needed (a partial of weight
        // 0 may hold NaN and must not reach the sum).
        const bool any_zero = __any_sync(kFull, j < cn && e == 0.f);
        for (int s0 = 0; s0 < cn; s0 += RC) {
            if (c > 0 || s0 > 0) {
#pragma unroll
                for (int i = 0; i < RC; ++i)
#pragma unroll
                    for (int k = 0; k < NV; ++k)
                        if (cl[k] && s0 + i < cn)
                            x[i][k] = ld_stream16(orow + (int64_t)(c + s0 + i) * p.o_r + k * p.lanes * 16);
            }
            auto fold_chunk = [&](auto check) {
#pragma unroll
                for (int i = 0; i < RC; ++i) {
                    const float w = __shfl_sync(kFull, e, s0 + i, p.lanes);
                    if (s0 + i < cn && (!decltype(check)::value || w != 0.f)) fold<TIn, NV, N2>(acc, x[i], w);
                }
            };
            if (any_zero) fold_chunk(std::true_type{});
            else fold_chunk(std::false_type{});
        }
    }
    esum = group_sum(esum, p.lanes);

    // esum >= 1 for a row with a finite max (its own weight is exp(0)).
    const float inv = esum > 0.f ? 1.f / esum : 0.f;
    store_cols<TOut, NV, N, N2>(p, ri.row, v0, live, acc, inv);
    if (live && ri.slice == 0 && j == 0) p.out_lse[ri.row] = esum > 0.f ? m + logf(esum) : -INFINITY;
}

// ------------------------------------------------------------------ stream kernel

// Persistent form of the vector kernel for R <= RC: each lane group walks
// the row slices grp, grp + G, grp + 2G, ... (G groups in the grid).  As soon
// as partial i of the current slice has been folded into the accumulator,
// its registers are refilled with partial i of the next slice, so every lane
// keeps up to R*NV 16-byte loads in flight across slice boundaries and no
// warp ever waits for a CTA to retire or launch.  FULL: R == RC, so no
// partial index needs a bound check.  A warp whose slices hold no empty
// shard folds every partial without a per-partial test (the common case);
// only a warp that has one checks each weight.  Measured on B200, back to
// back: R=16 B=512 H=16 D=512 24.6 -> 22.2 us, rank-major R=8 B=256 H=64
// D=128 7.7 -> 7.05 us (6.77 graph-replayed).  Refill loads of a column
// outside the next slice are skipped, not redirected: redirecting every
// lane's last refill to one shared address made a hot spot in L2 (30.2 us).
template <typename TIn, typename TOut, int RC, int NV, bool FULL>
__global__ void __launch_bounds__(kBlock, stream_min_blocks(RC, NV)) merge_stream_kernel(const KParams p, const int64_t G) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int j = (int)(t & (p.lanes - 1));
    // The first group of a warp has the most slices: a warp-uniform trip count
    // keeps every shuffle convergent; groups past their last slice idle.
    const int64_t grp0 = t >> p.lg;
    const int64_t grp_w = (t & ~(int64_t)31) >> p.lg;
    const int64_t trips = grp_w < p.groups ? (p.groups - grp_w + G - 1) / G : 0;
    const int R = FULL ? RC : p.R;

    struct Slice {
        const char* o;    // this lane's first column of partial 0
        const char* o0;   // column 0 of partial 0 of the row
        const float* l;
        int64_t row;
        int v0, slice;
        bool live;
        bool cl[NV];
    };
    auto locate = [&](int64_t g) {
        Slice s;
        s.live = g < p.groups;
        const RowIdx ri = row_of(p, s.live ? g : 0);
        s.row = ri.row;
        s.slice = ri.slice;
        s.v0 = ri.slice * p.lanes * NV + j;
#pragma unroll
        for (int k = 0; k < NV; ++k) s.cl[k] = s.live && s.v0 + k * p.lanes < p.dv;
        s.o0 = p.o + ri.b * p.o_b + ri.h * p.o_h;
        s.o = s.o0 + (int64_t)s.v0 * 16;
        s.l = p.lse + ri.b * p.l_b + ri.h * p.l_h;
        return s;
    };
    // Partial i of slice s into x[i] (the columns inside the slice).
    auto load = [&](uint4 (&xi)[NV], const Slice& s, int i) {
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (s.cl[k]) xi[k] = ld_stream16(s.o + (int64_t)i * p.o_r + k * p.lanes * 16);
    };

    Slice cur = locate(grp0);
    // The first kPrefetch slices' lines, while the previous grid drains.
    for (int64_t it = 0; it < kPrefetch && it < trips; ++it) {
        const Slice s = it == 0 ? cur : locate(grp0 + it * G);
#pragma unroll
        for (int i = 0; i < RC; ++i)
#pragma unroll
            for (int k = 0; k < NV; ++k)
                if (s.cl[k] && i < R) prefetch_l2(s.o + (int64_t)i * p.o_r + k * p.lanes * 16);
        if (s.live && j < R) prefetch_l2(s.l + (int64_t)j * p.l_r);
    }
    pdl_wait();
    pdl_release();
    // The first slice's loads go out without branches: a column outside the
    // slice reads column 0 of the same partial row instead (never used; a
    // different address for every row, so no L2 hot spot).  Measured:
    // R=16 B=512 H=16 D=512 22.6 -> 22.2 us graph-replayed.
    uint4 x[RC][NV];
#pragma unroll
    for (int i = 0; i < RC; ++i)
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            x[i][k] = make_uint4(0u, 0u, 0u, 0u);
            if (i < R)
                x[i][k] = ld_stream16((cur.cl[k] ? cur.o + k * p.lanes * 16 : cur.o0) + (int64_t)i * p.o_r);
        }
    float l = (cur.live && j < R) ? __ldg(cur.l + (int64_t)j * p.l_r) : -INFINITY;

    for (int64_t it = 0; it < trips; ++it) {
        const Slice nxt = locate(grp0 + (it + 1) * G);
        const float ln = (nxt.live && j < R) ? __ldg(nxt.l + (int64_t)j * p.l_r) : -INFINITY;

        const float m = group_max(l, p.lanes);
        const float mref = (m == -INFINITY) ? 0.f : m;
        const float e = expf(l - mref);
        const float esum = group_sum(e, p.lanes);
        const bool any_zero = __any_sync(kFull, j < R && e == 0.f);

        uint64_t acc[NV][N2];
#pragma unroll
        for (int k = 0; k < NV; ++k)
#pragma unroll
            for (int q = 0; q < N2; ++q) acc[k][q] = 0ull;
        // The two loops are written out: the generic-lambda form of the
        // other kernels measured 2-5 % slower here (rank-major R=8).
        if (!any_zero) {
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const float w = __shfl_sync(kFull, e, i, p.lanes);
                if (i < R) {
                    fold<TIn, NV, N2>(acc, x[i], w);
                    load(x[i], nxt, i);
                }
            }
        } else {
            // a partial of weight 0 may hold NaN: it must not reach the sum
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const float w = __shfl_sync(kFull, e, i, p.lanes);
                if (i < R) {
                    if (w != 0.f) fold<TIn, NV, N2>(acc, x[i], w);
                    load(x[i], nxt, i);
                }
            }
        }
        const float inv = esum > 0.f ? 1.f / esum : 0.f;
        store_cols<TOut, NV, N, N2>(p, cur.row, cur.v0, cur.live, acc, inv);
        if (cur.live && cur.slice == 0 && j == 0)
            p.out_lse[cur.row] = esum > 0.f ? m + logf(esum) : -INFINITY;
        cur = nxt;
        l = ln;
    }
}


// Persistent form for R > RC partials: the units a lane group walks are
// (row slice, chunk of RC partials) pairs -- chunk 0..nch-1 of slice grp,
// then of slice grp + G, ...  The group keeps a running (max M, weight sum,
// fp32 accumulator) over the chunks of its slice, rescaled by exp(M_old -
// M_new) when a chunk raises the max (the online form of the same LSE
// combine), and stores the slice after its last chunk.  As in the kernel
// above, partial i of the next unit is loaded into x[i] as soon as partial i
// of this unit is folded, so RC loads per lane stay in flight across chunk
// and slice boundaries.
template <typename TIn, typename TOut, int RC>
__global__ void __launch_bounds__(kBlock, stream_min_blocks(RC, 1)) merge_stream_long_kernel(const KParams p, const int64_t G) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int j = (int)(t & (p.lanes - 1));
    const int64_t grp0 = t >> p.lg;
    const int64_t grp_w = (t & ~(int64_t)31) >> p.lg;
    const int64_t trips = grp_w < p.groups ? (p.groups - grp_w + G - 1) / G : 0;
    const int nch = (p.R + RC - 1) / RC;   // chunks per slice, the same for every group

    struct Slice {
        const char* o;
        const float* l;
        int64_t row;
        int v, slice;
        bool live, cl;
    };
    auto locate = [&](int64_t g) {
        Slice s;
        s.live = g < p.groups;
        const RowIdx ri = row_of(p, s.live ? g : 0);
        s.row = ri.row;
        s.slice = ri.slice;
        s.v = ri.slice * p.lanes + j;
        s.cl = s.live && s.v < p.dv;
        s.o = p.o + ri.b * p.o_b + ri.h * p.o_h + (int64_t)s.v * 16;
        s.l = p.lse + ri.b * p.l_b + ri.h * p.l_h;
        return s;
    };
    // partial r0 + i of slice s (0 past the row's partials or the row)
    auto load_chunk = [&](const Slice& s, int r0, uint4 (&x)[RC]) {
#pragma unroll
        for (int i = 0; i < RC; ++i) {
            x[i] = make_uint4(0u, 0u, 0u, 0u);
            if (s.cl && r0 + i < p.R) x[i] = ld_stream16(s.o + (int64_t)(r0 + i) * p.o_r);
        }
    };
    auto load_lse = [&](const Slice& s, int r0) {
        return (s.live && j < RC && r0 + j < p.R) ? __ldg(s.l + (int64_t)(r0 + j) * p.l_r) : -INFINITY;
    };

    Slice cur = locate(grp0);
    if (kPrefetch && trips > 0) {   // the first chunk's lines, while the previous grid drains
#pragma unroll
        for (int i = 0; i < RC; ++i)
            if (cur.cl && i < p.R) prefetch_l2(cur.o + (int64_t)i * p.o_r);
        if (cur.live && j < RC && j < p.R) prefetch_l2(cur.l + (int64_t)j * p.l_r);
    }
    pdl_wait();
    pdl_release();
    uint4 x[RC];
    load_chunk(cur, 0, x);
    float l = load_lse(cur, 0);

    float M = -INFINITY, es = 0.f;
    uint64_t acc[N2];
#pragma unroll
    for (int q = 0; q < N2; ++q) acc[q] = 0ull;
    for (int64_t it = 0; it < trips; ++it) {
        for (int c = 0; c < nch; ++c) {
            const bool last = c + 1 == nch;
            const Slice nxt = last ? locate(grp0 + (it + 1) * G) : cur;
            const int rn = last ? 0 : (c + 1) * RC;   // first partial of the next unit
            const float ln = load_lse(nxt, rn);

            // fold chunk c: rescale the running state to the new max first
            const float Mn = fmaxf(M, group_max(l, p.lanes));
            const float ref = (Mn == -INFINITY) ? 0.f : Mn;   // all empty so far: no NaN
            const float sc = expf(M - ref);                   // 0 while the state is empty
            const uint64_t sc2 = pack2f(sc, sc);
#pragma unroll
            for (int q = 0; q < N2; ++q) mul2(acc[q], sc2);
            const float e = expf(l - ref);                    // 0 for an empty shard
            es = es * sc + group_sum(e, p.lanes);
            M = Mn;
            const int r0 = c * RC;
            const bool any_zero = __any_sync(kFull, j < RC && r0 + j < p.R && e == 0.f);
            // written out like the persistent kernel's (the generic-lambda
            // form measured 4 % slower at R=32)
            if (!any_zero) {
#pragma unroll
                for (int i = 0; i < RC; ++i) {
                    const float w = __shfl_sync(kFull, e, i, p.lanes);
                    if (r0 + i < p.R) {
                        uint64_t xx[N2];
                        Elem<TIn>::unpack2(x[i], xx);
                        const uint64_t ww = pack2f(w, w);
#pragma unroll
                        for (int q = 0; q < N2; ++q) fma2(acc[q], xx[q], ww);
                    }
                    x[i] = make_uint4(0u, 0u, 0u, 0u);
                    if (nxt.cl && rn + i < p.R) x[i] = ld_stream16(nxt.o + (int64_t)(rn + i) * p.o_r);
                }
            } else {
#pragma unroll
                for (int i = 0; i < RC; ++i) {
                    const float w = __shfl_sync(kFull, e, i, p.lanes);
                    if (r0 + i < p.R && w != 0.f) {
                        uint64_t xx[N2];
                        Elem<TIn>::unpack2(x[i], xx);
                        const uint64_t ww = pack2f(w, w);
#pragma unroll
                        for (int q = 0; q < N2; ++q) fma2(acc[q], xx[q], ww);
                    }
                    x[i] = make_uint4(0u, 0u, 0u, 0u);
                    if (nxt.cl && rn + i < p.R) x[i] = ld_stream16(nxt.o + (int64_t)(rn + i) * p.o_r);
                }
            }
            if (last) {
                const float inv = es > 0.f ? 1.f / es : 0.f;
                if (cur.cl) {
                    float f[N];
#pragma unroll
                    for (int q = 0; q < N2; ++q) {
                        unpack2f(acc[q], f[2 * q], f[2 * q + 1]);
                        f[2 * q] *= inv;
                        f[2 * q + 1] *= inv;
                    }
                    store_vec<TOut, N>(p.out + (cur.row * p.D + (int64_t)cur.v * N) * (int64_t)sizeof(TOut), f);
                }
                if (cur.live && cur.slice == 0 && j == 0)
                    p.out_lse[cur.row] = es > 0.f ? M + logf(es) : -INFINITY;
                M = -INFINITY;
                es = 0.f;
#pragma unroll
                for (int q = 0; q < N2; ++q) acc[q] = 0ull;
            }
            cur = nxt;
            l = ln;
        }
    }
}

// ------------------------------------------------------------------ wide kernel

// For R > 16, and for a handful of rows of any R (at most kWideMaxSlices row
// slices, where more threads per row beat more loads per thread): one CTA of
// up to kWideWarps warps per row slice, so that every partial of the row can
// be in flight at once.  The CTA's lane groups (of p.lanes lanes, one 16-byte
// column each) are S sub-groups; sub-group s takes the partials s, s + S,
// s + 2S, ... in batches of RC and keeps an online state (running max m,
// weight sum, fp32 accumulator), rescaled when a batch raises the max.  The S
// states are then merged -- the same LSE combine -- by shuffles inside each
// warp and through shared memory across warps.
constexpr int kWideWarps = 4;

__device__ __forceinline__ void combine_state(float& m, float& es, float* acc, float m2, float es2,
                                              const float* acc2, int n) {
    const float M = fmaxf(m, m2);
    const float Mref = (M == -INFINITY) ? 0.f : M;
    const float a = expf(m - Mref), a2 = expf(m2 - Mref);   // 0 for an empty state
    for (int k = 0; k < n; ++k) acc[k] = acc[k] * a + acc2[k] * a2;
    es = es * a + es2 * a2;
    m = M;
}

template <typename TIn, typename TOut, int RC>
__global__ void __launch_bounds__(kWideWarps * 32) merge_wide_kernel(const KParams p) {
    constexpr int N = Elem<TIn>::kVec;
    constexpr int N2 = N / 2;
    __shared__ float sh_acc[kWideWarps][32][N];
    __shared__ float sh_m[kWideWarps], sh_es[kWideWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = blockDim.x >> 5;                    // warps of this CTA (<= kWideWarps)
    const int j = lane & (p.lanes - 1);
    const int per_warp = 32 >> p.lg;                  // sub-groups per warp
    const int S = W * per_warp;
    const int s = warp * per_warp + (lane >> p.lg);
    const int s_w = warp * per_warp;                  // the warp's first sub-group: most partials
    const RowIdx ri = row_of(p, blockIdx.x);
    const int v = ri.slice * p.lanes + j;
    const bool vlive = v < p.dv;
    const char* orow = p.o + ri.b * p.o_b + ri.h * p.o_h + (int64_t)v * 16;
    const float* lrow = p.lse + ri.b * p.l_b + ri.h * p.l_h;
    const int n_w = p.R > s_w ? (p.R - s_w + S - 1) / S : 0;   // partials of sub-group s_w
    const int batches = (n_w + RC - 1) / RC;                    // warp-uniform
    if (kPrefetch) {   // the first batch, while the previous grid drains
#pragma unroll
        for (int i = 0; i < RC; ++i)
            if (vlive && s + S * i < p.R) prefetch_l2(orow + (int64_t)(s + S * i) * p.o_r);
        if (j < RC && s + S * j < p.R) prefetch_l2(lrow + (int64_t)(s + S * j) * p.l_r);
    }
    pdl_wait();
    pdl_release();

    float m = -INFINITY, es = 0.f;
    uint64_t acc[N2];
#pragma unroll
    for (int q = 0; q < N2; ++q) acc[q] = 0ull;
    for (int bt = 0; bt < batches; ++bt) {
        uint4 x[RC];
#pragma unroll
        for (int i = 0; i < RC; ++i) {
            const int r = s + S * (bt * RC + i);
            x[i] = make_uint4(0u, 0u, 0u, 0u);
            if (vlive && r < p.R) x[i] = ld_stream16(orow + (int64_t)r * p.o_r);
        }
        const int rj = s + S * (bt * RC + j);
        const float l = (j < RC && rj < p.R) ? __ldg(lrow + (int64_t)rj * p.l_r) : -INFINITY;
        const float mn = fmaxf(m, group_max(l, p.lanes));
        const float mref = (mn == -INFINITY) ? 0.f : mn;
        const float sc = expf(m - mref);   // rescale of the state so far (0 if it was empty)
#pragma unroll
        for (int q = 0; q < N2; ++q) {
            float a, b;
            unpack2f(acc[q], a, b);
            acc[q] = pack2f(a * sc, b * sc);
        }
        const float e = expf(l - mref);
        es = es * sc + group_sum(e, p.lanes);
        m = mn;
        const bool any_zero = __any_sync(kFull, j < RC && rj < p.R && e == 0.f);
        auto fold_chunk = [&](auto check) {
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const float w = __shfl_sync(kFull, e, i, p.lanes);
                const int r = s + S * (bt * RC + i);
                if (r < p.R && (!decltype(check)::value || w != 0.f)) {
                    uint64_t xx[N2];
                    Elem<TIn>::unpack2(x[i], xx);
                    const uint64_t ww = pack2f(w, w);
#pragma unroll
                    for (int q = 0; q < N2; ++q) fma2(acc[q], xx[q], ww);
                }
            }
        };
        if (any_zero) fold_chunk(std::true_type{});
        else fold_chunk(std::false_type{});
    }
    float f[N];
#pragma unroll
    for (int q = 0; q < N2; ++q) unpack2f(acc[q], f[2 * q], f[2 * q + 1]);
    // merge the sub-groups of this warp: partners differ in the lane bits above lg
    for (int off = p.lanes; off < 32; off <<= 1) {
        float f2[N];
#pragma unroll
        for (int k = 0; k < N; ++k) f2[k] = __shfl_xor_sync(kFull, f[k], off);
        const float m2 = __shfl_xor_sync(kFull, m, off);
        const float es2 = __shfl_xor_sync(kFull, es, off);
        combine_state(m, es, f, m2, es2, f2, N);
    }
    if (W > 1) {
        if (lane < p.lanes) {
#pragma unroll
            for (int k = 0; k < N; ++k) sh_acc[warp][lane][k] = f[k];
            if (lane == 0) {
                sh_m[warp] = m;
                sh_es[warp] = es;
            }
        }
        __syncthreads();
    }
    if (warp == 0 && lane < p.lanes) {
        for (int w = 1; w < W; ++w)
            combine_state(m, es, f, sh_m[w], sh_es[w], sh_acc[w][lane], N);
        const float inv = es > 0.f ? 1.f / es : 0.f;
#pragma unroll
        for (int k = 0; k < N; ++k) f[k] *= inv;
        if (vlive) store_vec<TOut, N>(p.out + (ri.row * p.D + (int64_t)v * N) * (int64_t)sizeof(TOut), f);
        if (ri.slice == 0 && lane == 0) p.out_lse[ri.row] = es > 0.f ? m + logf(es) : -INFINITY;
    }
}

// ------------------------------------------------------------------ scalar kernel

// Any alignment of strides and D: one warp per row, lane j handles the
// elements d = j, j+32, ...; element loads.
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kBlock) merge_scalar_kernel(const KParams p) {
    pdl_wait();
    pdl_release();
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = t >> 5;
    const int j = (int)(t & 31);
    const bool live = row < p.groups;
    const int64_t b = live ? row / p.H : 0, h = live ? row - b * p.H : 0;
    const char* orow = p.o + b * p.o_b + h * p.o_h;
    const float* lrow = p.lse + b * p.l_b + h * p.l_h;

    float m = -INFINITY;
    for (int c = 0; c < p.R; c += 32)
        if (live && c + j < p.R) m = fmaxf(m, __ldg(lrow + (int64_t)(c + j) * p.l_r));
    m = group_max(m, 32);
    const float mref = (m == -INFINITY) ? 0.f : m;

    float e0 = 0.f;
    if (live && j < p.R) e0 = expf(__ldg(lrow + (int64_t)j * p.l_r) - mref);
    float esum = e0;
    for (int c = 32; c < p.R; c += 32)
        if (live && c + j < p.R) esum += expf(__ldg(lrow + (int64_t)(c + j) * p.l_r) - mref);
    esum = group_sum(esum, 32);
    const float inv = esum > 0.f ? 1.f / esum : 0.f;

    for (int d0 = 0; d0 < p.D; d0 += 32) {
        const int d = d0 + j;
        const bool dlive = live && d < p.D;
        float acc = 0.f;
        for (int c = 0; c < p.R; c += 32) {
            float e = e0;
            if (c > 0) {
                e = 0.f;
                if (live && c + j < p.R) e = expf(__ldg(lrow + (int64_t)(c + j) * p.l_r) - mref);
            }
            const int cn = min(p.R - c, 32);
            for (int i = 0; i < cn; ++i) {
                const float w = __shfl_sync(kFull, e, i);
                if (dlive && w != 0.f)
                    acc = fmaf(w, Elem<TIn>::load1(orow + (int64_t)(c + i) * p.o_r +
                                                   (int64_t)d * (int64_t)sizeof(TIn)),
                               acc);
            }
        }
        if (dlive) Elem<TOut>::store1(p.out + (row * p.D + d) * (int64_t)sizeof(TOut), acc * inv);
    }
    if (live && j == 0) p.out_lse[row] = esum > 0.f ? m + logf(esum) : -INFINITY;
}


// ------------------------------------------------------------------ state update

struct SParams {
    char* acc;             // o_acc, dense [B,H,D]
    float* lse_acc;        // dense [B,H]
    const char* nw;        // o_new
    const float* lse_new;
    int64_t n_b, n_h;      // o_new strides in BYTES
    int64_t l_b, l_h;      // lse_new strides in elements
    int H, D, chunks;
    int lanes, lg;
    int64_t rows;
};

// 8 consecutive elements of type T at p as fp32; VEC: 16-byte accesses (p is
// 16-byte aligned and all 8 elements exist), else element accesses for the
// first `n`.  STREAM selects the read-only streaming load, only for data that
// this kernel never writes.
template <typename T, bool VEC, bool STREAM>
__device__ __forceinline__ void load8(const char* p, int n, float* f) {
    if constexpr (VEC) {
#pragma unroll
        for (int k = 0; k < (int)sizeof(T); k += 2) {   // 1 (16-bit) or 2 (fp32) vectors
            const uint4 v = STREAM ? ld_stream16(p + k * 8) : *reinterpret_cast<const uint4*>(p + k * 8);
            Elem<T>::unpack(v, f + k * 2);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            f[k] = 0.f;
            if (k < n) {
                if constexpr (STREAM) {
                    f[k] = Elem<T>::load1(p + k * (int)sizeof(T));
                } else if constexpr (sizeof(T) == 4) {
                    f[k] = *reinterpret_cast<const float*>(p + k * 4);
                } else {
                    f[k] = Elem<T>::widen(*reinterpret_cast<const unsigned short*>(p + k * 2));
                }
            }
        }
    }
}

template <typename T, bool VEC>
__device__ __forceinline__ void store8(char* p, int n, const float* f) {
    if constexpr (VEC) {
        store_vec<T, 8>(p, f);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < n) Elem<T>::store1(p + k * (int)sizeof(T), f[k]);
    }
}

// 8-element chunks a lane loads before it needs any weight: both sides of
// kStateChunks chunks are in flight while the two lse values arrive.
// Measured on B200 (B=512 H=16 D=512, fp32 accumulator, bf16 partial): one
// chunk 8.93 us (40 registers); two 10.11 us and four 11.03 us (more
// registers, fewer resident warps); loads issued only after the weights
// 10.04 us.
constexpr int kStateChunks = 1;
// Chunks per lane whose lines are prefetched into L2 before pdl_wait().
#ifndef LSEM_STATE_PREFETCH
#define LSEM_STATE_PREFETCH 4
#endif
constexpr int kStatePrefetch = LSEM_STATE_PREFETCH;

// A group of p.lanes lanes per row.  Lane 0 of the group reads both lse values
// and hands them to the group by shuffle, so no lane reads lse_acc after lane
// 0 has overwritten it; each element of o_acc is read and written by one lane.
// The data loads do not wait for the weights: a side of weight 0 is loaded
// but replaced by 0 before the FMA, so NaN stored there cannot reach the
// result.
template <typename TA, typename TN, bool VEC>
__global__ void __launch_bounds__(kBlock) state_update_kernel(const SParams p) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = t >> p.lg;
    const int j = (int)(t & (p.lanes - 1));
    const bool live = row < p.rows;
    const int64_t r = live ? row : 0;
    const int64_t b = r / p.H, h = r - b * p.H;
    char* arow = p.acc + r * p.D * (int64_t)sizeof(TA);
    const char* nrow = p.nw + b * p.n_b + h * p.n_h;
    if (kPrefetch && live) {   // this lane's first kStatePrefetch chunks of both sides
        for (int i = 0, c = j; i < kStatePrefetch && c < p.chunks; ++i, c += p.lanes) {
            prefetch_l2(arow + (int64_t)c * 8 * sizeof(TA));
            prefetch_l2(nrow + (int64_t)c * 8 * sizeof(TN));
        }
        if (j == 0) {
            prefetch_l2(p.lse_acc + r);
            prefetch_l2(p.lse_new + b * p.l_b + h * p.l_h);
        }
    }
    pdl_wait();
    pdl_release();

    float fa[kStateChunks][8], fn[kStateChunks][8];
    auto load_batch = [&](int c0) {
#pragma unroll
        for (int i = 0; i < kStateChunks; ++i) {
            const int c = c0 + i * p.lanes;
#pragma unroll
            for (int k = 0; k < 8; ++k) fa[i][k] = fn[i][k] = 0.f;
            if (live && c < p.chunks) {
                const int d0 = c * 8;
                const int n = min(8, p.D - d0);
                load8<TA, VEC, false>(arow + (int64_t)d0 * sizeof(TA), n, fa[i]);
                load8<TN, VEC, true>(nrow + (int64_t)d0 * sizeof(TN), n, fn[i]);
            }
        }
    };
    load_batch(j);

    float la = -INFINITY, ln = -INFINITY;
    if (live && j == 0) {
        la = p.lse_acc[r];
        ln = __ldg(p.lse_new + b * p.l_b + h * p.l_h);
    }
    la = __shfl_sync(kFull, la, 0, p.lanes);
    ln = __shfl_sync(kFull, ln, 0, p.lanes);
    const float m = fmaxf(la, ln);
    const float mref = (m == -INFINITY) ? 0.f : m;
    const float ea = expf(la - mref), en = expf(ln - mref);   // 0 for an empty side
    const float esum = ea + en;
    const float inv = esum > 0.f ? 1.f / esum : 0.f;
    if (!live) return;
    for (int c0 = j;;) {
#pragma unroll
        for (int i = 0; i < kStateChunks; ++i) {
            const int c = c0 + i * p.lanes;
            if (c < p.chunks) {
                const int d0 = c * 8;
                float o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float xa = ea != 0.f ? fa[i][k] : 0.f;
                    const float xn = en != 0.f ? fn[i][k] : 0.f;
                    o[k] = fmaf(ea, xa, en * xn) * inv;
                }
                store8<TA, VEC>(arow + (int64_t)d0 * sizeof(TA), min(8, p.D - d0), o);
            }
        }
        c0 += p.lanes * kStateChunks;
        if (c0 >= p.chunks) break;
        load_batch(c0);
    }
    if (j == 0) p.lse_acc[r] = esum > 0.f ? m + logf(esum) : -INFINITY;
}

using StateFn = void (*)(SParams);

template <typename TA, typename TN>
StateFn pick_state_v(bool vec) {
    return vec ? state_update_kernel<TA, TN, true> : state_update_kernel<TA, TN, false>;
}
template <typename TA>
StateFn pick_state_n(int new_dtype, bool vec) {
    switch (new_dtype) {
        case LSE_MERGE_F32: return pick_state_v<TA, float>(vec);
        case LSE_MERGE_F16: return pick_state_v<TA, __half>(vec);
        default: return pick_state_v<TA, __nv_bfloat16>(vec);
    }
}
StateFn pick_state(int acc_dtype, int new_dtype, bool vec) {
    switch (acc_dtype) {
        case LSE_MERGE_F32: return pick_state_n<float>(new_dtype, vec);
        case LSE_MERGE_F16: return pick_state_n<__half>(new_dtype, vec);
        default: return pick_state_n<__nv_bfloat16>(new_dtype, vec);
    }
}

// ------------------------------------------------------------------------ dispatch

using KernelFn = void (*)(KParams);
using StreamFn = void (*)(KParams, int64_t);

template <typename TIn, typename TOut>
StreamFn pick_long_rc(int rc) {
    return rc == 4 ? merge_stream_long_kernel<TIn, TOut, 4>
                   : rc == 8 ? merge_stream_long_kernel<TIn, TOut, 8> : merge_stream_long_kernel<TIn, TOut, 16>;
}
template <typename TIn>
StreamFn pick_long_out(int rc, int out_dtype) {
    switch (out_dtype) {
        case LSE_MERGE_F32: return pick_long_rc<TIn, float>(rc);
        case LSE_MERGE_F16: return pick_long_rc<TIn, __half>(rc);
        default: return pick_long_rc<TIn, __nv_bfloat16>(rc);
    }
}
StreamFn pick_stream_long(int rc, int in_dtype, int out_dtype) {
    switch (in_dtype) {
        case LSE_MERGE_F32: return pick_long_out<float>(rc, out_dtype);
        case LSE_MERGE_F16: return pick_long_out<__half>(rc, out_dtype);
        default: return pick_long_out<__nv_bfloat16>(rc, out_dtype);
    }
}

// (rc, nv) pairs the planner produces: rc * nv <= 16 loads of 16 bytes per lane.
// FULL instantiations serve R == rc.
template <typename TIn, typename TOut, bool FULL>
StreamFn pick_stream_kernel(int rc, int nv) {
    if constexpr (kMaxNv >= 4)
        if (rc == 4 && nv == 4) return merge_stream_kernel<TIn, TOut, 4, 4, FULL>;
    if (rc == 4) return nv == 2 ? merge_stream_kernel<TIn, TOut, 4, 2, FULL> : merge_stream_kernel<TIn, TOut, 4, 1, FULL>;
    if (rc == 8) return nv == 2 ? merge_stream_kernel<TIn, TOut, 8, 2, FULL> : merge_stream_kernel<TIn, TOut, 8, 1, FULL>;
    return merge_stream_kernel<TIn, TOut, 16, 1, FULL>;
}
template <typename TIn>
StreamFn pick_stream_out(int rc, int nv, bool full, int out_dtype) {
    switch (out_dtype) {
        case LSE_MERGE_F32: return full ? pick_stream_kernel<TIn, float, true>(rc, nv) : pick_stream_kernel<TIn, float, false>(rc, nv);
        case LSE_MERGE_F16: return full ? pick_stream_kernel<TIn, __half, true>(rc, nv) : pick_stream_kernel<TIn, __half, false>(rc, nv);
        default: return full ? pick_stream_kernel<TIn, __nv_bfloat16, true>(rc, nv)
                             : pick_stream_kernel<TIn, __nv_bfloat16, false>(rc, nv);
    }
}
StreamFn pick_stream(int rc, int nv, bool full, int in_dtype, int out_dtype) {
    switch (in_dtype) {
        case LSE_MERGE_F32: return pick_stream_out<float>(rc, nv, full, out_dtype);
        case LSE_MERGE_F16: return pick_stream_out<__half>(rc, nv, full, out_dtype);
        default: return pick_stream_out<__nv_bfloat16>(rc, nv, full, out_dtype);
    }
}

// CTAs of `fn` that fit on one SM of the current device, and its SM count;
// queried once per (device, kernel) and cached.
struct OccEntry {
    const void* fn;
    int dev, ctas, sms;
};
constexpr int kOccSlots = 512;
OccEntry g_occ[kOccSlots];
int g_occ_n = 0;
std::mutex g_occ_mu;

// Grid of a persistent kernel that would need `want_ctas` CTAs one-shot: at
// most what fits on the device at once.  With kBalance, when the last round
// of a full grid would be less than half full, the fewest CTAs that still
// need the same number of rounds, so no round is left mostly idle; a last
// round at least half full keeps the full grid, whose extra CTAs keep more
// loads in flight during the other rounds.  Measured on B200, back to back:
// R=16 B=512 H=16 D=512 (6.15 rounds): balanced 25.3 us, full 26.0 us;
// rank-major R=8 B=256 H=64 D=128 (1.73 rounds): full 7.3 us, balanced 7.8 us.
int64_t balanced(int64_t want_ctas, int64_t capacity) {
    if (want_ctas <= capacity) return want_ctas;
    if (!kBalance) return capacity;
    const int64_t rounds = (want_ctas + capacity - 1) / capacity;
    const int64_t last = want_ctas - (rounds - 1) * capacity;   // CTAs' worth of work in the last round
    if (2 * last >= capacity) return capacity;
    return (want_ctas + rounds - 1) / rounds;
}

int persistent_grid(const void* fn, int block, int64_t want_ctas, int* grid_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        for (int i = 0; i < g_occ_n; ++i)
            if (g_occ[i].fn == fn && g_occ[i].dev == dev) {
                *grid_out = (int)balanced(want_ctas, (int64_t)g_occ[i].ctas * g_occ[i].sms);
                return 0;
            }
    }
    int ctas = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas, fn, block, 0);
    if (e != cudaSuccess) return (int)e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return (int)e;
    if (ctas < 1) ctas = 1;
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        if (g_occ_n < kOccSlots) g_occ[g_occ_n++] = OccEntry{fn, dev, ctas, sms};
    }
    *grid_out = (int)balanced(want_ctas, (int64_t)ctas * sms);
    return 0;
}

template <typename TIn, typename TOut>
KernelFn pick_kernel(const lse_merge_plan& pl) {
    if (pl.path == LSE_MERGE_PATH_SCALAR) return merge_scalar_kernel<TIn, TOut>;
    if (pl.path == LSE_MERGE_PATH_WIDE)
        return pl.rc == 4 ? merge_wide_kernel<TIn, TOut, 4>
                          : pl.rc == 8 ? merge_wide_kernel<TIn, TOut, 8> : merge_wide_kernel<TIn, TOut, 16>;
    const int rc = pl.rc, nv = pl.nv;
    if (rc == 4) return nv == 4 ? merge_vec_kernel<TIn, TOut, 4, 4>
                      : nv == 2 ? merge_vec_kernel<TIn, TOut, 4, 2> : merge_vec1_kernel<TIn, TOut, 4>;
    if (rc == 8) return nv == 2 ? merge_vec_kernel<TIn, TOut, 8, 2> : merge_vec1_kernel<TIn, TOut, 8>;
    return merge_vec1_kernel<TIn, TOut, 16>;
}

template <typename TIn>
KernelFn pick_out(const lse_merge_plan& pl, int out_dtype) {
    switch (out_dtype) {
        case LSE_MERGE_F32: return pick_kernel<TIn, float>(pl);
        case LSE_MERGE_F16: return pick_kernel<TIn, __half>(pl);
        default: return pick_kernel<TIn, __nv_bfloat16>(pl);
    }
}

KernelFn pick(const lse_merge_plan& pl, int in_dtype, int out_dtype) {
    switch (in_dtype) {
        case LSE_MERGE_F32: return pick_out<float>(pl, out_dtype);
        case LSE_MERGE_F16: return pick_out<__half>(pl, out_dtype);
        default: return pick_out<__nv_bfloat16>(pl, out_dtype);
    }
}


int log2i(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return l;
}

int run(const void* partial_o, const float* partial_lse, int R, int B, int H, int D,
        const lse_merge_strides* strides, int in_dtype, int out_dtype, void* out_o,
        float* out_lse, cudaStream_t stream, int path) {
    if (R < 1 || B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    const lse_merge_strides st = strides ? *strides : default_strides(R, B, H, D);
    lse_merge_plan pl;
    const int rc = make_plan(partial_o, partial_lse, R, B, H, D, st, in_dtype, out_dtype, out_o,
                             out_lse, path, &pl);
    if (rc != LSE_MERGE_OK) return rc;

    const int ib = elem_bytes(in_dtype);
    KParams kp;
    kp.o = static_cast<const char*>(partial_o);
    kp.lse = partial_lse;
    kp.out = static_cast<char*>(out_o);
    kp.out_lse = out_lse;
    kp.o_r = st.o_r * ib;
    kp.o_b = st.o_b * ib;
    kp.o_h = st.o_h * ib;
    kp.l_r = st.lse_r;
    kp.l_b = st.lse_b;
    kp.l_h = st.lse_h;
    kp.R = R;
    kp.H = H;
    kp.D = D;
    kp.dv = pl.path == LSE_MERGE_PATH_SCALAR ? D : D / pl.vec;
    kp.lanes = pl.lanes;
    kp.lg = log2i(pl.lanes);
    kp.spr = pl.slices_per_row;
    kp.groups = pl.groups;
    kp.idx32 = (pl.groups < ((int64_t)1 << 32)) ? 1 : 0;
    kp.c_spr = fastdiv_c((uint32_t)pl.slices_per_row);
    kp.c_H = fastdiv_c((uint32_t)H);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3((unsigned)pl.block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    const bool pdl = kPdl != 0;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e;
    if (pl.path == LSE_MERGE_PATH_STREAM) {
        const StreamFn fn = R > pl.rc ? pick_stream_long(pl.rc, in_dtype, out_dtype)
                                      : pick_stream(pl.rc, pl.nv, R == pl.rc, in_dtype, out_dtype);
        const int64_t want = (pl.groups * pl.lanes + pl.block - 1) / pl.block;
        int grid = 0;
        const int qe = persistent_grid((const void*)fn, pl.block, want, &grid);
        if (qe != 0) {
            set_last_cuda_error(qe);
            (void)cudaGetLastError();
            return LSE_MERGE_ELAUNCH;
        }
        cfg.gridDim = dim3((unsigned)grid);
        const int64_t G = (int64_t)grid * pl.block / pl.lanes;
        e = cudaLaunchKernelEx(&cfg, fn, kp, G);
    } else {
        e = cudaLaunchKernelEx(&cfg, pick(pl, in_dtype, out_dtype), kp);
    }
    if (e != cudaSuccess) {
        set_last_cuda_error((int)e);
        (void)cudaGetLastError();  // the failure belongs to this call; do not leave it pending
        return LSE_MERGE_ELAUNCH;
    }
    return LSE_MERGE_OK;
}

int run_state(void* o_acc, float* lse_acc, const void* o_new, const float* lse_new, int B,
              int H, int D, const lse_merge_state_strides* strides, int acc_dtype, int new_dtype,
              cudaStream_t stream) {
    if (B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    lse_merge_state_strides st;
    if (strides) {
        st = *strides;
    } else {
        st.o_b = (int64_t)H * D;
        st.o_h = D;
        st.lse_b = H;
        st.lse_h = 1;
    }
    StatePlan pl;
    const int rc = make_state_plan(o_acc, lse_acc, o_new, lse_new, B, H, D, st, acc_dtype,
                                   new_dtype, &pl);
    if (rc != LSE_MERGE_OK) return rc;
    const int nb = elem_bytes(new_dtype);
    SParams sp;
    sp.acc = static_cast<char*>(o_acc);
    sp.lse_acc = lse_acc;
    sp.nw = static_cast<const char*>(o_new);
    sp.lse_new = lse_new;
    sp.n_b = st.o_b * nb;
    sp.n_h = st.o_h * nb;
    sp.l_b = st.lse_b;
    sp.l_h = st.lse_h;
    sp.H = H;
    sp.D = D;
    sp.chunks = pl.chunks;
    sp.lanes = pl.lanes;
    sp.lg = log2i(pl.lanes);
    sp.rows = (int64_t)B * H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3((unsigned)pl.block);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = kPdl ? attr : nullptr;
    cfg.numAttrs = kPdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, pick_state(acc_dtype, new_dtype, pl.vec != 0), sp);
    if (e != cudaSuccess) {
        set_last_cuda_error((int)e);
        (void)cudaGetLastError();
        return LSE_MERGE_ELAUNCH;
    }
    return LSE_MERGE_OK;
}

}  // namespace
}  // namespace lsem

extern "C" {

int lse_merge(const void* partial_o, const float* partial_lse, int R, int B, int H, int D,
              const lse_merge_strides* strides, int in_dtype, int out_dtype, void* out_o,
              float* out_lse, lse_merge_stream_t stream) {
    return lsem::run(partial_o, partial_lse, R, B, H, D, strides, in_dtype, out_dtype, out_o,
                     out_lse, reinterpret_cast<cudaStream_t>(stream), LSE_MERGE_PATH_AUTO);
}

int lse_merge_with_path(const void* partial_o, const float* partial_lse, int R, int B, int H,
                        int D, const lse_merge_strides* strides, int in_dtype, int out_dtype,
                        void* out_o, float* out_lse, lse_merge_stream_t stream, int path) {
    return lsem::run(partial_o, partial_lse, R, B, H, D, strides, in_dtype, out_dtype, out_o,
                     out_lse, reinterpret_cast<cudaStream_t>(stream), path);
}

int lse_merge_state_update(void* o_acc, float* lse_acc, const void* o_new, const float* lse_new,
                           int B, int H, int D, const lse_merge_state_strides* new_strides,
                           int acc_dtype, int new_dtype, lse_merge_stream_t stream) {
    return lsem::run_state(o_acc, lse_acc, o_new, lse_new, B, H, D, new_strides, acc_dtype,
                           new_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int lse_merge_last_cuda_error(void) { return lsem::last_cuda_error(); }

}  // extern "C"
