/*
 * oracle_threads.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * Runs the unchanged fp64 oracle merge (oracle_lse_merge in
 * lse_merge_oracle.c) on several host threads at once, for timing the CPU
 * baseline on every core of a machine.  It does no arithmetic of the method:
 * it cuts the batch axis into contiguous ranges, one per thread, and calls
 * oracle_lse_merge on each range with its pointers moved to the range's first
 * batch.  Rows are independent in the merge, so the result is bit-identical
 * to one call over all batches.
 */
#include <pthread.h>
#include <stdint.h>
#include <unistd.h>

int oracle_lse_merge(const void* partial_o, const float* partial_lse,
                     int R, int B, int H, int D,
                     const int64_t* os, const int64_t* ls, int in_dtype,
                     double* out_o, double* out_lse);

struct range_job {
    const char* o;
    const float* lse;
    int R, B, H, D, in_dtype;
    const int64_t* os;
    const int64_t* ls;
    double* out_o;
    double* out_lse;
    int rc;
};

static void* run_range(void* arg) {
    struct range_job* j = (struct range_job*)arg;
    j->rc = oracle_lse_merge(j->o, j->lse, j->R, j->B, j->H, j->D, j->os, j->ls, j->in_dtype,
                             j->out_o, j->out_lse);
    return 0;
}

/* Number of threads oracle_lse_merge_threads uses for `threads` <= 0. */
int oracle_host_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * The same arguments and result as oracle_lse_merge, computed by
 * min(threads, B) threads (threads <= 0: one per online core).  Returns the
 * first non-zero code of a range, -3 if a thread could not be started, and
 * writes the number of threads used to *used when `used` is not NULL.
 */
int oracle_lse_merge_threads(const void* partial_o, const float* partial_lse,
                             int R, int B, int H, int D,
                             const int64_t* os, const int64_t* ls, int in_dtype,
                             double* out_o, double* out_lse, int threads, int* used) {
    enum { MAX_THREADS = 1024 };
    if (R < 1 || B < 1 || H < 1 || D < 1) return -2;
    if (threads <= 0) threads = oracle_host_threads();
    if (threads > B) threads = B;
    if (threads > MAX_THREADS) threads = MAX_THREADS;
    const int64_t esize = in_dtype == 0 ? 4 : 2;
    struct range_job jobs[MAX_THREADS];
    pthread_t tid[MAX_THREADS];
    int started = 0, rc = 0;
    for (int t = 0; t < threads; ++t) {
        const int b0 = (int)((int64_t)B * t / threads), b1 = (int)((int64_t)B * (t + 1) / threads);
        struct range_job* j = &jobs[t];
        j->o = (const char*)partial_o + (int64_t)b0 * os[1] * esize;
        j->lse = partial_lse + (int64_t)b0 * ls[1];
        j->R = R;
        j->B = b1 - b0;
        j->H = H;
        j->D = D;
        j->in_dtype = in_dtype;
        j->os = os;
        j->ls = ls;
        j->out_o = out_o + (int64_t)b0 * H * D;
        j->out_lse = out_lse + (int64_t)b0 * H;
        j->rc = 0;
        if (pthread_create(&tid[t], 0, run_range, j) != 0) {
            rc = -3;
            break;
        }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        pthread_join(tid[t], 0);
        if (rc == 0 && jobs[t].rc != 0) rc = jobs[t].rc;
    }
    if (used) *used = started;
    return rc;
}
