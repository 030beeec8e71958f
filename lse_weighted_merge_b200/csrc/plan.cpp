// plan.cpp -- validation and launch geometry of the LSE-weighted merge.
//
// Geometry of the vector kernels (the merge of one (b,h) row is spread over
// a group of `lanes` consecutive lanes of one warp):
//   * vec     = 16 bytes / element size: one 16-byte column of a row;
//   * rc      = 4, 8 or 16 partial rows loaded before the first FMA;
//   * nv      = 16-byte columns per lane in each partial row, 16 / rc, halved
//               while it would leave fewer than rc lanes with work, so that a
//               lane keeps rc * nv <= 16 loads (256 bytes) in flight;
//   * lanes   = the power of two >= D / (vec * nv) (at most 32), and at least
//               rc so the lanes of a group hold one lse value each per batch;
//   * slices  = ceil((D/vec) / (lanes * nv)) groups per row.
// The latency path is the same kernel launched as one CTA of exactly the
// threads needed, for problems of at most kLatencyMaxThreads threads.
#include "plan.h"

#include <cstdint>

namespace lsem {

namespace {
thread_local int g_last_cuda_error = 0;
}
void set_last_cuda_error(int e) { g_last_cuda_error = e; }
int last_cuda_error() { return g_last_cuda_error; }

int elem_bytes(int dtype) {
    switch (dtype) {
        case LSE_MERGE_F32: return 4;
        case LSE_MERGE_F16: return 2;
        case LSE_MERGE_BF16: return 2;
        default: return 0;
    }
}

lse_merge_strides default_strides(int R, int B, int H, int D) {
    (void)B;
    lse_merge_strides s;
    s.o_r = D;
    s.o_b = (int64_t)H * R * D;
    s.o_h = (int64_t)R * D;
    s.lse_r = 1;
    s.lse_b = (int64_t)H * R;
    s.lse_h = R;
    return s;
}

namespace {

using i128 = __int128;

// Byte interval [lo, hi) of a buffer.
struct Span {
    uintptr_t lo;
    i128 hi;
};

bool overlap(const Span& a, const Span& b) {
    return (i128)a.lo < b.hi && (i128)b.lo < a.hi;
}

int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

bool aligned(const void* p, int a) { return ((uintptr_t)p % (uintptr_t)a) == 0; }

}  // namespace

int make_plan(const void* o, const float* lse, int R, int B, int H, int D,
              const lse_merge_strides& st, int in_dtype, int out_dtype, const void* out_o,
              const float* out_lse, int path, lse_merge_plan* plan) {
    const int ib = elem_bytes(in_dtype), ob = elem_bytes(out_dtype);
    if (ib == 0 || ob == 0) return LSE_MERGE_EDTYPE;
    if (R < 1 || B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    if (!o || !lse || !out_o || !out_lse || !plan) return LSE_MERGE_ENULL;
    if (st.o_r < 0 || st.o_b < 0 || st.o_h < 0 || st.lse_r < 0 || st.lse_b < 0 || st.lse_h < 0)
        return LSE_MERGE_ESTRIDE;
    if (path < LSE_MERGE_PATH_AUTO || path > LSE_MERGE_PATH_WIDE) return LSE_MERGE_EPATH;
    if (!aligned(o, ib) || !aligned(out_o, ob) || !aligned(lse, 4) || !aligned(out_lse, 4))
        return LSE_MERGE_EALIGN;

    // Extents in bytes, in 128-bit arithmetic so that no product can wrap.
    const i128 o_last = (i128)(R - 1) * st.o_r + (i128)(B - 1) * st.o_b + (i128)(H - 1) * st.o_h + D;
    const i128 l_last = (i128)(R - 1) * st.lse_r + (i128)(B - 1) * st.lse_b + (i128)(H - 1) * st.lse_h + 1;
    const i128 rows = (i128)B * H;
    const i128 lim = (i128)1 << 62;
    const i128 o_bytes = o_last * ib, l_bytes = l_last * 4, out_bytes = rows * D * ob, ol_bytes = rows * 4;
    if (o_bytes > lim || l_bytes > lim || out_bytes > lim || ol_bytes > lim) return LSE_MERGE_EDIMS;

    const Span so{(uintptr_t)o, (i128)(uintptr_t)o + o_bytes};
    const Span sl{(uintptr_t)lse, (i128)(uintptr_t)lse + l_bytes};
    const Span su{(uintptr_t)out_o, (i128)(uintptr_t)out_o + out_bytes};
    const Span sv{(uintptr_t)out_lse, (i128)(uintptr_t)out_lse + ol_bytes};
    if (overlap(su, so) || overlap(su, sl) || overlap(sv, so) || overlap(sv, sl) || overlap(su, sv))
        return LSE_MERGE_EALIAS;

    // Can the 16-byte vector kernels take these arguments?
    const int vec = 16 / ib;
    const int out_align = (vec * ob) < 16 ? vec * ob : 16;
    const bool vec_ok = (D % vec) == 0 && aligned(o, 16) && ((st.o_r * ib) % 16) == 0 &&
                        ((st.o_b * ib) % 16) == 0 && ((st.o_h * ib) % 16) == 0 &&
                        aligned(out_o, out_align);

    lse_merge_plan p{};
    if (vec_ok && path != LSE_MERGE_PATH_SCALAR) {
        const int dv = D / vec;
        int rc = R <= 4 ? 4 : (R <= 8 ? 8 : 16);
        // lanes and slices for nv columns per lane
        auto shape = [&](int nv, int* lanes, int* slices) {
            const int cols = (dv + nv - 1) / nv;
            *lanes = next_pow2(cols < 32 ? cols : 32);
            if (*lanes < rc) *lanes = rc;
            *slices = (dv + *lanes * nv - 1) / (*lanes * nv);
        };
        // The latency path (one CTA) keeps one column per lane: for a
        // problem that small, more threads beat more loads per thread.
        int lanes1, slices1;
        shape(1, &lanes1, &slices1);
        const bool small = rows * slices1 * lanes1 <= kLatencyMaxThreads;
        // STREAM takes a row slice's partials in one batch when R <= rc, and
        // in chunks of 16 with a running max (the long form) beyond.
        const i128 in_bytes = (i128)R * rows * D * ib;
        int chosen = path;
        if (chosen == LSE_MERGE_PATH_AUTO) {
            if (small)
                chosen = LSE_MERGE_PATH_LATENCY;
            else if (rows * slices1 <= kWideMaxSlices)
                chosen = LSE_MERGE_PATH_WIDE;
            else if (R > rc) {
                // the long form when its lanes (one column each) fill most of
                // a wave; otherwise WIDE, which also spreads a row's partials
                // over the warps of a CTA
                const int lanes_d = next_pow2(dv < 32 ? dv : 32);
                const i128 threads = rows * ((dv + lanes_d - 1) / lanes_d) * (lanes_d < 4 ? 4 : lanes_d);
                chosen = kAutoStreamLong && threads >= kLongMinThreads ? LSE_MERGE_PATH_STREAM
                                                                       : LSE_MERGE_PATH_WIDE;
            }
            else if (kAutoStream && in_bytes >= kStreamMinBytes && in_bytes <= kStreamMaxBytes)
                chosen = LSE_MERGE_PATH_STREAM;
            else
                chosen = LSE_MERGE_PATH_VECTOR;
        }
        if (chosen == LSE_MERGE_PATH_LATENCY && !small) return LSE_MERGE_EPATH;
        if (chosen == LSE_MERGE_PATH_WIDE) {
            // One 16-byte column per lane, at least 4 lanes.  Just enough
            // warps (at most 4) that the lane groups hold every partial of the
            // row in one batch of at most min(16, lanes) per group; the batch
            // size rc then shrinks to what the groups need (a power of two >= 4).
            int lanes = next_pow2(dv < 32 ? dv : 32);
            if (lanes < 4) lanes = 4;
            const int rc_max = lanes < 16 ? lanes : 16;
            const int per_warp = 32 / lanes;
            int warps = (R + rc_max * per_warp - 1) / (rc_max * per_warp);
            if (warps > kWideBlock / 32) warps = kWideBlock / 32;
            const int groups_cta = warps * per_warp;
            int rc = next_pow2((R + groups_cta - 1) / groups_cta);
            if (rc < 4) rc = 4;
            if (rc > rc_max) rc = rc_max;
            p.path = chosen;
            p.vec = vec;
            p.lanes = lanes;
            p.rc = rc;
            p.nv = 1;
            p.slices_per_row = (dv + lanes - 1) / lanes;
            p.groups = (int64_t)(rows * p.slices_per_row);
            p.block = warps * 32;
            if ((i128)p.groups > 0x7fffffff) return LSE_MERGE_EDIMS;
            p.grid = p.groups;
            *plan = p;
            return LSE_MERGE_OK;
        }
        int nv = 1;
        if (chosen == LSE_MERGE_PATH_STREAM && R > rc) {
            // the long form: chunks of as many partials as a row has
            // 16-byte columns (4..16), one column per lane
            const int lanes_d = next_pow2(dv < 32 ? dv : 32);
            rc = lanes_d < 4 ? 4 : (lanes_d > 16 ? 16 : lanes_d);
        } else if (chosen != LSE_MERGE_PATH_LATENCY) {
            nv = 16 / rc < kMaxNv ? 16 / rc : kMaxNv;
            while (nv > 1 && (dv + nv - 1) / nv < rc) nv >>= 1;
        }
        int lanes, slices;
        shape(nv, &lanes, &slices);
        const i128 groups = rows * slices;
        const i128 threads = groups * lanes;
        p.path = chosen;
        p.vec = vec;
        p.lanes = lanes;
        p.rc = rc;
        p.nv = nv;
        p.slices_per_row = slices;
        p.groups = (int64_t)groups;
        if (chosen == LSE_MERGE_PATH_LATENCY) {
            p.block = (int)((threads + 31) / 32 * 32);
            p.grid = 1;
        } else if (chosen == LSE_MERGE_PATH_STREAM) {
            p.block = kBlock;
            p.grid = 0;   // persistent: sized at launch from the device's occupancy
        } else {
            p.block = kBlock;
            const i128 grid = (threads + kBlock - 1) / kBlock;
            if (grid > 0x7fffffff) return LSE_MERGE_EDIMS;
            p.grid = (int64_t)grid;
        }
    } else {
        if (path == LSE_MERGE_PATH_VECTOR || path == LSE_MERGE_PATH_LATENCY ||
            path == LSE_MERGE_PATH_STREAM || path == LSE_MERGE_PATH_WIDE)
            return LSE_MERGE_EPATH;
        p.path = LSE_MERGE_PATH_SCALAR;
        p.vec = 1;
        p.lanes = 32;
        p.rc = 0;
        p.nv = 1;
        p.slices_per_row = 1;
        p.groups = (int64_t)rows;
        p.block = kBlock;
        const i128 grid = (rows * 32 + kBlock - 1) / kBlock;
        if (grid > 0x7fffffff) return LSE_MERGE_EDIMS;
        p.grid = (int64_t)grid;
    }
    *plan = p;
    return LSE_MERGE_OK;
}

lse_merge_attn_strides default_attn_strides(int Hq, int Hkv, int L, int D) {
    lse_merge_attn_strides s;
    s.q_b = (int64_t)Hq * D;
    s.q_h = D;
    s.k_b = s.v_b = (int64_t)Hkv * L * D;
    s.k_h = s.v_h = (int64_t)L * D;
    s.k_l = s.v_l = D;
    return s;
}

int attn_workspace_layout(int B, int Hq, int Hkv, int R, int D, AttnPlan* plan) {
    if (B < 1 || Hq < 1 || Hkv < 1 || R < 1 || D < 1 || Hq % Hkv != 0) return LSE_MERGE_EDIMS;
    const auto up = [](i128 x) { return (x + 255) / 256 * 256; };
    const i128 rows = (i128)B * Hq * R;   // = B * Hkv * R * G
    const i128 l_off = up((i128)B * Hkv * 4);
    const i128 o_off = up(l_off + rows * 4);
    const i128 total = o_off + rows * D * 4;
    if (total > ((i128)1 << 62)) return LSE_MERGE_EDIMS;
    plan->ws_l_off = (int64_t)l_off;
    plan->ws_o_off = (int64_t)o_off;
    plan->ws_bytes = (int64_t)total;
    return LSE_MERGE_OK;
}

// out_o / out_lse: the merged outputs (fused modes) or the partial buffers
// (dense [B,Hq,R,D] and [B,Hq,R] fp32) of the unfused producer.
int make_attn_plan(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int L,
                   int D, int R, float scale, const lse_merge_attn_strides& st, int dtype,
                   int out_dtype, const void* out_o, const float* out_lse, int mode,
                   const void* ws, int64_t ws_bytes, AttnPlan* plan) {
    const int fused = mode != kAttnModePartials;
    const int ob = elem_bytes(out_dtype);
    if (elem_bytes(dtype) == 0 || ob == 0) return LSE_MERGE_EDTYPE;
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || D < 1 || R < 1) return LSE_MERGE_EDIMS;
    if (!q || !k || !v || !out_o || !out_lse || !plan) return LSE_MERGE_ENULL;
    if (st.q_b < 0 || st.q_h < 0 || st.k_b < 0 || st.k_h < 0 || st.k_l < 0 || st.v_b < 0 ||
        st.v_h < 0 || st.v_l < 0)
        return LSE_MERGE_ESTRIDE;
    if (dtype == LSE_MERGE_F32) return LSE_MERGE_EUNSUP;
    if (D != 64 && D != 128) return LSE_MERGE_EUNSUP;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return LSE_MERGE_EUNSUP;
    if (mode == kAttnModeCluster && R != 1 && R != 2 && R != 4 && R != 8) return LSE_MERGE_EUNSUP;
    if (mode == kAttnModeWorkspace && !ws) return LSE_MERGE_ENULL;
    if (B > 65535 || Hkv > 65535 || R > 65535) return LSE_MERGE_EDIMS;
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return LSE_MERGE_EDIMS;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out_o, ob) ||
        !aligned(out_lse, 4))
        return LSE_MERGE_EALIGN;
    const int64_t s16[8] = {st.q_b, st.q_h, st.k_b, st.k_h, st.k_l, st.v_b, st.v_h, st.v_l};
    for (int i = 0; i < 8; ++i)
        if ((s16[i] * 2) % 16 != 0) return LSE_MERGE_EALIGN;
    const i128 lim = (i128)1 << 62;
    const i128 q_bytes = ((i128)(B - 1) * st.q_b + (i128)(Hq - 1) * st.q_h + D) * 2;
    const i128 k_bytes = ((i128)(B - 1) * st.k_b + (i128)(Hkv - 1) * st.k_h + (i128)(L - 1) * st.k_l + D) * 2;
    const i128 v_bytes = ((i128)(B - 1) * st.v_b + (i128)(Hkv - 1) * st.v_h + (i128)(L - 1) * st.v_l + D) * 2;
    const i128 rows = (i128)B * Hq;
    const i128 o_bytes = fused ? rows * D * ob : rows * R * D * 4;
    const i128 l_bytes = fused ? rows * 4 : rows * R * 4;
    if (q_bytes > lim || k_bytes > lim || v_bytes > lim || o_bytes > lim || l_bytes > lim)
        return LSE_MERGE_EDIMS;
    const Span sq{(uintptr_t)q, (i128)(uintptr_t)q + q_bytes};
    const Span sk{(uintptr_t)k, (i128)(uintptr_t)k + k_bytes};
    const Span sv{(uintptr_t)v, (i128)(uintptr_t)v + v_bytes};
    const Span so{(uintptr_t)out_o, (i128)(uintptr_t)out_o + o_bytes};
    const Span sl{(uintptr_t)out_lse, (i128)(uintptr_t)out_lse + l_bytes};
    if (overlap(so, sq) || overlap(so, sk) || overlap(so, sv) || overlap(sl, sq) ||
        overlap(sl, sk) || overlap(sl, sv) || overlap(so, sl))
        return LSE_MERGE_EALIAS;
    AttnPlan p{};
    p.G = Hq / Hkv;
    p.mode = mode;
    if (mode == kAttnModeWorkspace) {
        const int lrc = attn_workspace_layout(B, Hq, Hkv, R, D, &p);
        if (lrc != LSE_MERGE_OK) return lrc;
        if (!aligned(ws, 16)) return LSE_MERGE_EALIGN;
        if (ws_bytes < p.ws_bytes) return LSE_MERGE_EDIMS;
        const Span sw{(uintptr_t)ws, (i128)(uintptr_t)ws + p.ws_bytes};
        if (overlap(sw, sq) || overlap(sw, sk) || overlap(sw, sv) || overlap(sw, so) ||
            overlap(sw, sl))
            return LSE_MERGE_EALIAS;
    }
    const int64_t ring = (int64_t)kAttnWarps * kAttnStages * 2 * kAttnTileKeys * D * 2;
    // after the key loop the ring is reused for each warp's state (G <= 16
    // rows of m, l and D accumulators; sized for 16)
    const int64_t states = (int64_t)kAttnWarps * 16 * (D + 2) * 4;
    const int64_t base = ((ring > states ? ring : states) + 15) / 16 * 16;
    // fused: behind them CTA 0's receive buffer of the R split partials (an
    // mbarrier, lse [R][G] padded to 4 floats, o [R][G][D]), which siblings
    // fill while CTA 0 may still use its ring
    const int64_t rg = (int64_t)R * p.G;
    p.smem = base;
    // cluster: CTA 0's receive buffer behind the ring
    if (mode == kAttnModeCluster) p.smem = base + 16 + ((rg + 3) & ~(int64_t)3) * 4 + rg * D * 4;
    if (p.smem > kAttnMaxSmem) return LSE_MERGE_EUNSUP;
    *plan = p;
    return LSE_MERGE_OK;
}

int make_state_plan(const void* o_acc, const float* lse_acc, const void* o_new,
                    const float* lse_new, int B, int H, int D, const lse_merge_state_strides& st,
                    int acc_dtype, int new_dtype, StatePlan* plan) {
    const int ab = elem_bytes(acc_dtype), nb = elem_bytes(new_dtype);
    if (ab == 0 || nb == 0) return LSE_MERGE_EDTYPE;
    if (B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    if (!o_acc || !lse_acc || !o_new || !lse_new || !plan) return LSE_MERGE_ENULL;
    if (st.o_b < 0 || st.o_h < 0 || st.lse_b < 0 || st.lse_h < 0) return LSE_MERGE_ESTRIDE;
    if (!aligned(o_acc, ab) || !aligned(o_new, nb) || !aligned(lse_acc, 4) || !aligned(lse_new, 4))
        return LSE_MERGE_EALIGN;
    const i128 rows = (i128)B * H;
    const i128 lim = (i128)1 << 62;
    const i128 acc_bytes = rows * D * ab, lacc_bytes = rows * 4;
    const i128 new_bytes = ((i128)(B - 1) * st.o_b + (i128)(H - 1) * st.o_h + D) * nb;
    const i128 lnew_bytes = ((i128)(B - 1) * st.lse_b + (i128)(H - 1) * st.lse_h + 1) * 4;
    if (acc_bytes > lim || new_bytes > lim || lnew_bytes > lim) return LSE_MERGE_EDIMS;
    const Span sa{(uintptr_t)o_acc, (i128)(uintptr_t)o_acc + acc_bytes};
    const Span sla{(uintptr_t)lse_acc, (i128)(uintptr_t)lse_acc + lacc_bytes};
    const Span sn{(uintptr_t)o_new, (i128)(uintptr_t)o_new + new_bytes};
    const Span sln{(uintptr_t)lse_new, (i128)(uintptr_t)lse_new + lnew_bytes};
    if (overlap(sa, sla) || overlap(sa, sn) || overlap(sa, sln) || overlap(sla, sn) ||
        overlap(sla, sln))
        return LSE_MERGE_EALIAS;
    StatePlan p{};
    p.vec = (D % 8) == 0 && aligned(o_acc, 16) && aligned(o_new, 16) && ((st.o_b * nb) % 16) == 0 &&
            ((st.o_h * nb) % 16) == 0;
    p.chunks = (D + 7) / 8;
    p.lanes = next_pow2(p.chunks < 32 ? p.chunks : 32);
    p.block = kBlock;
    const i128 grid = (rows * p.lanes + kBlock - 1) / kBlock;
    if (grid > 0x7fffffff) return LSE_MERGE_EDIMS;
    p.grid = (int64_t)grid;
    *plan = p;
    return LSE_MERGE_OK;
}

int cp_layout(int world, int B, int H, int D, int in_dtype, CpPlan* plan) {
    const int ib = elem_bytes(in_dtype);
    if (ib == 0) return LSE_MERGE_EDTYPE;
    if (world < 1 || world > LSE_MERGE_CP_MAX_WORLD || B < 1 || H < 1 || D < 1 || H % world != 0)
        return LSE_MERGE_EDIMS;
    if (((int64_t)D * ib) % 16 != 0) return LSE_MERGE_EALIGN;
    const i128 lim = (i128)1 << 62;
    const int Hq = H / world;
    const i128 slot_o = (i128)B * Hq * D * ib, slot_l = (i128)B * Hq * 4;
    const i128 n = 2 * (i128)(world - 1);
    const auto up = [](i128 x) { return (x + 255) / 256 * 256; };
    const i128 o_off = kCpHeaderBytes;
    const i128 l_off = up(o_off + n * slot_o);
    const i128 total = up(l_off + n * slot_l);
    if ((i128)B * H * D * ib > lim || total > lim) return LSE_MERGE_EDIMS;
    // every 16-byte unit index of the kernel fits in 31 bits (32 GiB of
    // partials per rank)
    if ((i128)world * B * (H / world) * (D * ib / 16) >= ((i128)1 << 31)) return LSE_MERGE_EDIMS;
    CpPlan p{};
    p.world = world;
    p.Hq = Hq;
    p.in_bytes = ib;
    p.dv = (int)((int64_t)D * ib / 16);
    p.U = (int64_t)B * Hq * p.dv;
    p.slot_o = (int64_t)slot_o;
    p.slot_l = (int64_t)slot_l;
    p.o_off = (int64_t)o_off;
    p.l_off = (int64_t)l_off;
    p.ws_bytes = (int64_t)total;
    *plan = p;
    return LSE_MERGE_OK;
}

int make_cp_plan(const lse_merge_cp_args& a, CpPlan* plan) {
    const int ob = elem_bytes(a.out_dtype);
    if (elem_bytes(a.in_dtype) == 0 || ob == 0) return LSE_MERGE_EDTYPE;
    CpPlan p{};
    int rc = cp_layout(a.world, a.B, a.H, a.D, a.in_dtype, &p);
    if (rc != LSE_MERGE_OK) return rc;
    if (a.rank_begin < 0 || a.rank_count < 1 || a.rank_begin + a.rank_count > a.world)
        return LSE_MERGE_EDIMS;
    if (a.timeout_ns <= 0 || a.timeout_ns > kCpMaxTimeoutNs) return LSE_MERGE_EDIMS;
    if (a.flags & ~(LSE_MERGE_CP_FLAG_CROSS_GPU_PROTOCOL | LSE_MERGE_CP_FLAG_TEST_SILENT_LAST_RANK))
        return LSE_MERGE_EDIMS;
    p.rank_begin = a.rank_begin;
    p.rank_count = a.rank_count;
    p.out_bytes = ob;
    const i128 in_o = (i128)a.B * a.H * a.D * p.in_bytes, in_l = (i128)a.B * a.H * 4;
    const i128 out_o = (i128)a.B * p.Hq * a.D * ob, out_l = (i128)a.B * p.Hq * 4;
    // Written spans (workspaces, outputs) may overlap nothing else; inputs
    // are only read and may overlap one another.
    Span wr[3 * LSE_MERGE_CP_MAX_WORLD], rd[2 * LSE_MERGE_CP_MAX_WORLD];
    int nw = 0, nr = 0;
    for (int q = 0; q < a.world; ++q) {
        if (!a.ws[q]) return LSE_MERGE_ENULL;
        if (!aligned(a.ws[q], 256)) return LSE_MERGE_EALIGN;
        wr[nw++] = Span{(uintptr_t)a.ws[q], (i128)(uintptr_t)a.ws[q] + p.ws_bytes};
    }
    for (int i = 0; i < a.rank_count; ++i) {
        if (!a.local_o[i] || !a.local_lse[i] || !a.out_o[i] || !a.out_lse[i]) return LSE_MERGE_ENULL;
        if (!aligned(a.local_o[i], 16) || !aligned(a.out_o[i], 16) || !aligned(a.local_lse[i], 4) ||
            !aligned(a.out_lse[i], 4))
            return LSE_MERGE_EALIGN;
        rd[nr++] = Span{(uintptr_t)a.local_o[i], (i128)(uintptr_t)a.local_o[i] + in_o};
        rd[nr++] = Span{(uintptr_t)a.local_lse[i], (i128)(uintptr_t)a.local_lse[i] + in_l};
        wr[nw++] = Span{(uintptr_t)a.out_o[i], (i128)(uintptr_t)a.out_o[i] + out_o};
        wr[nw++] = Span{(uintptr_t)a.out_lse[i], (i128)(uintptr_t)a.out_lse[i] + out_l};
    }
    for (int i = 0; i < nw; ++i) {
        for (int j = i + 1; j < nw; ++j)
            if (overlap(wr[i], wr[j])) return LSE_MERGE_EALIAS;
        for (int j = 0; j < nr; ++j)
            if (overlap(wr[i], rd[j])) return LSE_MERGE_EALIAS;
    }
    *plan = p;
    return LSE_MERGE_OK;
}

}  // namespace lsem

extern "C" {

int lse_merge_cp_workspace_bytes(int world, int B, int H, int D, int in_dtype, int64_t* bytes) {
    if (!bytes) return LSE_MERGE_ENULL;
    lsem::CpPlan p;
    const int rc = lsem::cp_layout(world, B, H, D, in_dtype, &p);
    if (rc == LSE_MERGE_OK) *bytes = p.ws_bytes;
    return rc;
}

int lse_merge_cp_validate(const lse_merge_cp_args* args) {
    if (!args) return LSE_MERGE_ENULL;
    lsem::CpPlan p;
    return lsem::make_cp_plan(*args, &p);
}

int lse_merge_decode_workspace_bytes(int B, int Hq, int Hkv, int R, int D, int64_t* bytes) {
    if (!bytes) return LSE_MERGE_ENULL;
    lsem::AttnPlan p{};
    const int rc = lsem::attn_workspace_layout(B, Hq, Hkv, R, D, &p);
    if (rc == LSE_MERGE_OK) *bytes = p.ws_bytes;
    return rc;
}

int lse_merge_plan_query(const void* partial_o, const float* partial_lse, int R, int B, int H,
                         int D, const lse_merge_strides* strides, int in_dtype, int out_dtype,
                         const void* out_o, const float* out_lse, int path,
                         lse_merge_plan* plan) {
    if (R < 1 || B < 1 || H < 1 || D < 1) return LSE_MERGE_EDIMS;
    const lse_merge_strides st = strides ? *strides : lsem::default_strides(R, B, H, D);
    return lsem::make_plan(partial_o, partial_lse, R, B, H, D, st, in_dtype, out_dtype, out_o,
                           out_lse, path, plan);
}

const char* lse_merge_strerror(int code) {
    switch (code) {
        case LSE_MERGE_OK: return "ok";
        case LSE_MERGE_EDTYPE: return "unknown element type (in_dtype/out_dtype)";
        case LSE_MERGE_EDIMS: return "R, B, H and D must be >= 1 and the extents must fit";
        case LSE_MERGE_ENULL: return "a required pointer is NULL";
        case LSE_MERGE_ESTRIDE: return "strides must be >= 0";
        case LSE_MERGE_EALIAS: return "an output overlaps an input or the other output";
        case LSE_MERGE_ELAUNCH: return "CUDA kernel launch failed";
        case LSE_MERGE_EALIGN: return "a pointer is not aligned to its element size";
        case LSE_MERGE_EPATH: return "the requested kernel path cannot take these arguments";
        case LSE_MERGE_EUNSUP: return "shape not implemented by the decode-attention kernels (dtype, D, group, R)";
        case LSE_MERGE_ECUDA: return "a CUDA runtime call of a set-up function failed";
        case LSE_MERGE_ESCRATCH: return "the problem needs more scratch or staging memory than the library's array or the host context holds";
        case LSE_MERGE_EDEVICE: return "the current device is not the one the host context was made on";
        default: return "unknown lse_merge error code";
    }
}

int lse_merge_version(void) { return LSE_MERGE_ABI_VERSION; }

}  // extern "C"
