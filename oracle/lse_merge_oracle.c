/*
 * lse_merge_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, obviously correct CPU statement of the LSE-weighted merge,
 * in fp64.  Only the test suite, the smoke check in __graft_entry__.py and
 * bench.py's CPU-baseline / reference arm may load this library.  The CUDA
 * path shares no code, header, table or helper with it and never calls it.
 *
 * What the method computes comes from the page
 *   "[flashinfer] FlashInfer의 Context-Parallel Decode 최적화: Fused A2A + LSE Reduce"
 *   (an analysis of FlashInfer PR #4929):
 *   - section "들어가며" (introduction): under context-parallel decode the KV
 *     cache is split along the sequence; each rank runs attention over its own
 *     KV shard and produces a partial output o_r plus lse_r, the log-sum-exp
 *     normaliser of that shard's scores.
 *   - section "코드 분석 / 1. Fused Kernel 구현" (the Before/After snippet):
 *     the legacy merge upcasts the partials to fp32, multiplies them by
 *     weights, sums over the partial axis (dim -2 of a [..., R, D] tensor)
 *     and divides by denom; the fused kernel's steps 2 and 3 are "LSE-based
 *     softmax weights" and "accumulate in FP32, then convert to FP16/BF16".
 *
 * Readings where the page is silent:
 *   - lse is a natural logarithm;
 *   - weights = exp(lse_r - m) with m = max_r lse_r, denom = sum of weights
 *     (the plainest reading of the snippet's `weights` and `denom`);
 *   - lse_r = -inf marks an empty shard: weight 0 and its o_r is not read;
 *   - a row whose shards are all empty gives out = 0 and merged lse = -inf;
 *   - merged lse = m + log(denom);
 *   - lse = +inf or NaN is outside the domain: the result is whatever the
 *     fp64 arithmetic below gives (NaN propagates), nothing is special-cased.
 *
 * The result stays in fp64; rounding to the output dtype is not modelled.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Element types, numbered like the public C-ABI but defined here on their own. */
enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

int oracle_version(void) { return 1; }

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double widen_f16(uint16_t bits) {
    int sign = bits >> 15;
    int e = (bits >> 10) & 0x1f;
    int f = bits & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^(1-15-10) */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
static double widen_bf16(uint16_t bits) {
    int sign = bits >> 15;
    int e = (bits >> 7) & 0xff;
    int f = bits & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);                /* subnormal: f * 2^(1-127-7) */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);     /* (1 + f/2^7) * 2^(e-127) */
    return sign ? -v : v;
}

static double widen_f32(const void* p) {
    float x;
    memcpy(&x, p, sizeof x);
    return (double)x;
}

/* Exact value of one stored element, widened to double. */
static double load_elem(const void* base, int64_t idx, int dtype) {
    if (dtype == ORACLE_F32)
        return widen_f32((const char*)base + idx * 4);
    uint16_t bits;
    memcpy(&bits, (const char*)base + idx * 2, sizeof bits);
    return dtype == ORACLE_F16 ? widen_f16(bits) : widen_bf16(bits);
}

/* Exposed so the tests can check the decoders against library conversions. */
double oracle_widen(uint32_t bits, int dtype) {
    if (dtype == ORACLE_F16) return widen_f16((uint16_t)bits);
    if (dtype == ORACLE_BF16) return widen_bf16((uint16_t)bits);
    float x;
    memcpy(&x, &bits, sizeof x);
    return (double)x;
}

/*
 * The merge.  For every row (b, h):
 *     m       = max_r lse_r
 *     e_r     = exp(lse_r - m)            (0 for an empty shard, lse_r = -inf)
 *     denom   = sum_r e_r
 *     out[d]  = (sum_r e_r * o_r[d]) / denom
 *     out_lse = m + log(denom)
 * and out = 0, out_lse = -inf when every shard of the row is empty.
 *
 * partial_o   element (r, b, h, d) at index r*os[0] + b*os[1] + h*os[2] + d
 * partial_lse element (r, b, h)    at index r*ls[0] + b*ls[1] + h*ls[2]
 * out_o       double [B, H, D], contiguous
 * out_lse     double [B, H], contiguous
 * Returns 0, or -1 for an unknown dtype, -2 for a non-positive size.
 */
int oracle_lse_merge(const void* partial_o, const float* partial_lse,
                     int R, int B, int H, int D,
                     const int64_t* os, const int64_t* ls, int in_dtype,
                     double* out_o, double* out_lse) {
    if (in_dtype != ORACLE_F32 && in_dtype != ORACLE_F16 && in_dtype != ORACLE_BF16)
        return -1;
    if (R < 1 || B < 1 || H < 1 || D < 1)
        return -2;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int64_t o_row = (int64_t)b * os[1] + (int64_t)h * os[2];
            const int64_t l_row = (int64_t)b * ls[1] + (int64_t)h * ls[2];
            double* out = out_o + ((int64_t)b * H + h) * D;
            double* olse = out_lse + (int64_t)b * H + h;

            double m = -INFINITY;
            for (int r = 0; r < R; ++r) {
                double l = (double)partial_lse[l_row + (int64_t)r * ls[0]];
                if (l > m) m = l;
            }
            if (m == -INFINITY) {                       /* every shard empty */
                for (int d = 0; d < D; ++d) out[d] = 0.0;
                *olse = -INFINITY;
                continue;
            }

            for (int d = 0; d < D; ++d) out[d] = 0.0;
            double denom = 0.0;
            for (int r = 0; r < R; ++r) {
                double l = (double)partial_lse[l_row + (int64_t)r * ls[0]];
                if (l == -INFINITY) continue;           /* empty shard: weight 0, o_r not read */
                double e = exp(l - m);
                denom += e;
                const int64_t o_sh = o_row + (int64_t)r * os[0];
                for (int d = 0; d < D; ++d)
                    out[d] += e * load_elem(partial_o, o_sh + d, in_dtype);
            }
            for (int d = 0; d < D; ++d) out[d] /= denom;
            *olse = m + log(denom);
        }
    }
    return 0;
}

/*
 * Softmax attention of one query over the keys [begin, end) of one KV shard,
 * the producer of a partial (the introduction of the same page: each rank
 * attends over its local KV shard and returns o_r and lse_r).
 *     s_j = scale * <q, k_j>
 *     lse = log sum_j exp(s_j)          (evaluated as mx + log sum_j exp(s_j - mx))
 *     o   = sum_j exp(s_j - lse) * v_j
 * An empty key range gives o = 0 and lse = -inf.
 * q: [D]; k, v: [L, D] row-major; o: [D].
 */
void oracle_attention_shard(const double* q, const double* k, const double* v,
                            int L, int D, double scale, int begin, int end,
                            double* o, double* lse) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (begin < 0) begin = 0;
    if (end > L) end = L;
    if (end <= begin) {
        *lse = -INFINITY;
        return;
    }
    double mx = -INFINITY;
    for (int j = begin; j < end; ++j) {
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += q[d] * k[(int64_t)j * D + d];
        s *= scale;
        if (s > mx) mx = s;
    }
    double z = 0.0;
    for (int j = begin; j < end; ++j) {
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += q[d] * k[(int64_t)j * D + d];
        s *= scale;
        double p = exp(s - mx);
        z += p;
        for (int d = 0; d < D; ++d) o[d] += p * v[(int64_t)j * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= z;
    *lse = mx + log(z);
}

/*
 * Fold one new partial into an accumulator: the merge above with R = 2, the
 * first partial being the accumulator (the combine the page's merge is built
 * from; applying it shard by shard gives the R-way merge, by associativity of
 * the log-sum-exp combine).  Per row (b, h):
 *     m   = max(lse_acc, lse_new)
 *     e_a = exp(lse_acc - m), e_n = exp(lse_new - m)   (0 for an lse of -inf)
 *     out = (e_a * acc + e_n * new) / (e_a + e_n),  out_lse = m + log(e_a + e_n)
 * and 0, -inf when both are empty.  acc is dense [B, H, D] of acc_dtype with
 * lse_acc dense [B, H]; new has element strides nb, nh (d stride 1) and lse_new
 * strides lb, lh.  Results in fp64: out [B, H, D], out_lse [B, H].
 */
int oracle_state_update(const void* acc, const float* lse_acc, int acc_dtype,
                        const void* nw, const float* lse_new, int new_dtype,
                        int B, int H, int D, int64_t nb, int64_t nh, int64_t lb, int64_t lh,
                        double* out, double* out_lse) {
    if ((acc_dtype != ORACLE_F32 && acc_dtype != ORACLE_F16 && acc_dtype != ORACLE_BF16) ||
        (new_dtype != ORACLE_F32 && new_dtype != ORACLE_F16 && new_dtype != ORACLE_BF16))
        return -1;
    if (B < 1 || H < 1 || D < 1) return -2;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int64_t row = (int64_t)b * H + h;
            const double la = (double)lse_acc[row];
            const double ln = (double)lse_new[(int64_t)b * lb + (int64_t)h * lh];
            double* o = out + row * D;
            const double m = la > ln ? la : ln;
            if (m == -INFINITY) {
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                out_lse[row] = -INFINITY;
                continue;
            }
            const double ea = (la == -INFINITY) ? 0.0 : exp(la - m);
            const double en = (ln == -INFINITY) ? 0.0 : exp(ln - m);
            const double denom = ea + en;
            for (int d = 0; d < D; ++d) {
                double s = 0.0;
                if (ea != 0.0) s += ea * load_elem(acc, row * D + d, acc_dtype);
                if (en != 0.0) s += en * load_elem(nw, (int64_t)b * nb + (int64_t)h * nh + d, new_dtype);
                o[d] = s / denom;
            }
            out_lse[row] = m + log(denom);
        }
    }
    return 0;
}

/*
 * Context-parallel exchange followed by the merge (page "[flashinfer]
 * FlashInfer의 Context-Parallel Decode 최적화: Fused A2A + LSE Reduce",
 * sections "들어가며" and "코드 분석 / 1. Fused Kernel 구현": every rank holds
 * the partials of its KV shard for all heads; the exchange hands each head to
 * the rank that owns it, which then merges the partials of all ranks).
 * Reading: heads are scattered in equal contiguous blocks, rank q owning heads
 * [q*H/world, (q+1)*H/world).  So rank q's output row (b, j) is the merge over
 * ranks s of rank s's partial at (b, q*H/world + j):
 *     out[q][b][j] = merge_s (local_o[s][b][q*Hq + j], local_lse[s][b][q*Hq + j])
 * local_o     [world, B, H, D] elements of in_dtype, contiguous
 * local_lse   [world, B, H] float, contiguous
 * out_o       double [world, B, H/world, D];  out_lse  double [world, B, H/world]
 * Returns 0, -1 for an unknown dtype, -2 for a bad size (H % world != 0).
 */
int oracle_cp_exchange_merge(const void* local_o, const float* local_lse, int world,
                             int B, int H, int D, int in_dtype,
                             double* out_o, double* out_lse) {
    if (in_dtype != ORACLE_F32 && in_dtype != ORACLE_F16 && in_dtype != ORACLE_BF16)
        return -1;
    if (world < 1 || B < 1 || H < 1 || D < 1 || H % world != 0) return -2;
    const int Hq = H / world;
    const int64_t esize = in_dtype == ORACLE_F32 ? 4 : 2;
    const int64_t os[3] = {(int64_t)B * H * D, (int64_t)H * D, D};
    const int64_t ls[3] = {(int64_t)B * H, H, 1};
    for (int q = 0; q < world; ++q) {
        const int64_t h0 = (int64_t)q * Hq;             /* first head rank q owns */
        const char* o = (const char*)local_o + h0 * D * esize;
        const float* l = local_lse + h0;
        int rc = oracle_lse_merge(o, l, world, B, Hq, D, os, ls, in_dtype,
                                  out_o + (int64_t)q * B * Hq * D, out_lse + (int64_t)q * B * Hq);
        if (rc != 0) return rc;
    }
    return 0;
}
