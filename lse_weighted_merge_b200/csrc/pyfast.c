/* pyfast.c -- a CPython extension that forwards the per-call entry points
 * of liblse_merge.so with vectorcall argument passing.
 *
 * It adds no behaviour: each function converts its Python integers to the C
 * types of include/lse_merge.h and calls the library, which validates the
 * arguments and launches the kernel.  It exists because a ctypes call with a
 * dozen arguments costs several microseconds of marshalling, more than the
 * launch itself for a small merge; the ctypes binding (_native.py) keeps
 * every other call.
 *
 *   merge(o, lse, R, B, H, D, strides, in_dtype, out_dtype, out, out_lse,
 *         stream, path) -> int        lse_merge_with_path; strides is None or
 *                                      (o_r, o_b, o_h, lse_r, lse_b, lse_h)
 *   state_update(acc, lse_acc, new, lse_new, B, H, D, strides, acc_dtype,
 *                new_dtype, stream) -> int
 *                                      lse_merge_state_update; strides is None
 *                                      or (o_b, o_h, lse_b, lse_h)
 *   cp_exchange_merge(args_address, stream) -> int
 *                                      lse_merge_cp_exchange_merge on an
 *                                      lse_merge_cp_args the caller owns
 * Pointers and the stream are integers (0 for NULL / the legacy stream).  The
 * return value is the library's code; nothing raises on a library error.
 */
#define PY_SSIZE_T_CLEAN
#include <Python.h>
#include <stdint.h>

#include "lse_merge.h"

static int as_i64(PyObject* o, long long* v) {
    *v = PyLong_AsLongLong(o);
    return (*v == -1 && PyErr_Occurred()) ? -1 : 0;
}

static int as_int(PyObject* o, int* v) {
    long long x;
    if (as_i64(o, &x)) return -1;
    if (x < INT32_MIN || x > INT32_MAX) {
        PyErr_SetString(PyExc_OverflowError, "size or code does not fit a C int");
        return -1;
    }
    *v = (int)x;
    return 0;
}

static int as_ptr(PyObject* o, void** p) {
    if (o == Py_None) {
        *p = NULL;
        return 0;
    }
    unsigned long long x = PyLong_AsUnsignedLongLong(o);
    if (x == (unsigned long long)-1 && PyErr_Occurred()) return -1;
    *p = (void*)(uintptr_t)x;
    return 0;
}

/* A tuple of n integers into out[0..n-1]; returns 1 for None, 0 when filled. */
static int as_i64_tuple(PyObject* o, int64_t* out, Py_ssize_t n) {
    if (o == Py_None) return 1;
    if (!PyTuple_Check(o) || PyTuple_GET_SIZE(o) != n) {
        PyErr_Format(PyExc_TypeError, "strides must be None or a tuple of %zd integers", n);
        return -1;
    }
    for (Py_ssize_t i = 0; i < n; ++i) {
        long long v;
        if (as_i64(PyTuple_GET_ITEM(o, i), &v)) return -1;
        out[i] = (int64_t)v;
    }
    return 0;
}

static int nargs_ok(Py_ssize_t n, Py_ssize_t want, const char* name) {
    if (n == want) return 1;
    PyErr_Format(PyExc_TypeError, "%s takes %zd arguments (%zd given)", name, want, n);
    return 0;
}

static PyObject* fast_merge(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (!nargs_ok(n, 13, "merge")) return NULL;
    void *o, *lse, *out, *out_lse, *stream;
    int R, B, H, D, in_dtype, out_dtype, path;
    int64_t s[6];
    if (as_ptr(a[0], &o) || as_ptr(a[1], &lse) || as_int(a[2], &R) || as_int(a[3], &B) ||
        as_int(a[4], &H) || as_int(a[5], &D))
        return NULL;
    const int st = as_i64_tuple(a[6], s, 6);
    if (st < 0) return NULL;
    if (as_int(a[7], &in_dtype) || as_int(a[8], &out_dtype) || as_ptr(a[9], &out) ||
        as_ptr(a[10], &out_lse) || as_ptr(a[11], &stream) || as_int(a[12], &path))
        return NULL;
    lse_merge_strides strides = {s[0], s[1], s[2], s[3], s[4], s[5]};
    int rc;
    Py_BEGIN_ALLOW_THREADS
    rc = lse_merge_with_path(o, (const float*)lse, R, B, H, D, st == 0 ? &strides : NULL,
                             in_dtype, out_dtype, out, (float*)out_lse,
                             (lse_merge_stream_t)stream, path);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(rc);
}

static PyObject* fast_state_update(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (!nargs_ok(n, 11, "state_update")) return NULL;
    void *acc, *lse_acc, *nw, *lse_new, *stream;
    int B, H, D, acc_dtype, new_dtype;
    int64_t s[4];
    if (as_ptr(a[0], &acc) || as_ptr(a[1], &lse_acc) || as_ptr(a[2], &nw) ||
        as_ptr(a[3], &lse_new) || as_int(a[4], &B) || as_int(a[5], &H) || as_int(a[6], &D))
        return NULL;
    const int st = as_i64_tuple(a[7], s, 4);
    if (st < 0) return NULL;
    if (as_int(a[8], &acc_dtype) || as_int(a[9], &new_dtype) || as_ptr(a[10], &stream))
        return NULL;
    lse_merge_state_strides strides = {s[0], s[1], s[2], s[3]};
    int rc;
    Py_BEGIN_ALLOW_THREADS
    rc = lse_merge_state_update(acc, (float*)lse_acc, nw, (const float*)lse_new, B, H, D,
                                st == 0 ? &strides : NULL, acc_dtype, new_dtype,
                                (lse_merge_stream_t)stream);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(rc);
}

static PyObject* fast_cp(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (!nargs_ok(n, 2, "cp_exchange_merge")) return NULL;
    void *args, *stream;
    if (as_ptr(a[0], &args) || as_ptr(a[1], &stream)) return NULL;
    int rc;
    Py_BEGIN_ALLOW_THREADS
    rc = lse_merge_cp_exchange_merge((const lse_merge_cp_args*)args, (lse_merge_stream_t)stream);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(rc);
}

static PyMethodDef fast_methods[] = {
    {"merge", (PyCFunction)(void (*)(void))fast_merge, METH_FASTCALL,
     "lse_merge_with_path(o, lse, R, B, H, D, strides, in_dtype, out_dtype, out, out_lse, stream, path)"},
    {"state_update", (PyCFunction)(void (*)(void))fast_state_update, METH_FASTCALL,
     "lse_merge_state_update(acc, lse_acc, new, lse_new, B, H, D, strides, acc_dtype, new_dtype, stream)"},
    {"cp_exchange_merge", (PyCFunction)(void (*)(void))fast_cp, METH_FASTCALL,
     "lse_merge_cp_exchange_merge(args_address, stream)"},
    {NULL, NULL, 0, NULL},
};

static struct PyModuleDef fast_module = {
    PyModuleDef_HEAD_INIT, "_fast",
    "Vectorcall forwarding of liblse_merge.so's per-call entry points.", -1, fast_methods,
    NULL, NULL, NULL, NULL,
};

PyMODINIT_FUNC PyInit__fast(void) { return PyModule_Create(&fast_module); }
