/* _qmm_call -- the per-call hand-off of qmm() from Python to the C ABI, in C.
 *
 * A ctypes call converts every argument through Python-level descriptors, which costs
 * several microseconds per call: as much as a whole small-M matmul on the GPU.  This module
 * takes the same plain integers (device pointers, sizes, format, plan address, stream
 * handle) as a vectorcall and forwards them to the library's qmm_ex, whose address the
 * Python side binds once from the loaded libqmm_b200.so.  It does no arithmetic and holds no
 * state beyond that one function pointer; all argument checks stay in the library.
 */
#define PY_SSIZE_T_CLEAN
#include <Python.h>
#include <stdint.h>

typedef int (*qmm_ex_fn)(const void* x, const uint32_t* packed, const uint16_t* scales,
                         const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K,
                         int bits, int group, int dtype, const void* plan, void* stream);

static qmm_ex_fn g_qmm_ex = NULL;

static PyObject* bind(PyObject* self, PyObject* arg) {
    (void)self;
    void* p = PyLong_AsVoidPtr(arg);
    if (p == NULL) {
        if (!PyErr_Occurred()) PyErr_SetString(PyExc_ValueError, "qmm_ex address is null");
        return NULL;
    }
    g_qmm_ex = (qmm_ex_fn)p;
    Py_RETURN_NONE;
}

/* qmm_ex(x, packed, scales, biases, y, M, N, K, bits, group, dtype, plan, stream) -> status
 * Pointers, the plan address (0 = default plan) and the stream handle are Python ints. */
static PyObject* call(PyObject* self, PyObject* const* args, Py_ssize_t nargs) {
    (void)self;
    if (nargs != 13) {
        PyErr_SetString(PyExc_TypeError, "qmm_ex takes 13 arguments");
        return NULL;
    }
    if (g_qmm_ex == NULL) {
        PyErr_SetString(PyExc_RuntimeError, "qmm_ex is not bound");
        return NULL;
    }
    void* ptr[5];
    for (int i = 0; i < 5; ++i) ptr[i] = PyLong_AsVoidPtr(args[i]);
    const long long M = PyLong_AsLongLong(args[5]);
    const long long N = PyLong_AsLongLong(args[6]);
    const long long K = PyLong_AsLongLong(args[7]);
    const long bits = PyLong_AsLong(args[8]);
    const long group = PyLong_AsLong(args[9]);
    const long dtype = PyLong_AsLong(args[10]);
    void* plan = PyLong_AsVoidPtr(args[11]);
    void* stream = PyLong_AsVoidPtr(args[12]);
    if (PyErr_Occurred()) return NULL;
    const int st = g_qmm_ex(ptr[0], (const uint32_t*)ptr[1], (const uint16_t*)ptr[2],
                            (const uint16_t*)ptr[3], ptr[4], (int64_t)M, (int64_t)N, (int64_t)K,
                            (int)bits, (int)group, (int)dtype, plan, stream);
    return PyLong_FromLong(st);
}

static PyMethodDef methods[] = {
    {"bind", bind, METH_O, "bind(address of qmm_ex)"},
    {"qmm_ex", (PyCFunction)(void (*)(void))call, METH_FASTCALL,
     "qmm_ex(x, packed, scales, biases, y, M, N, K, bits, group, dtype, plan, stream) -> status"},
    {NULL, NULL, 0, NULL},
};

static struct PyModuleDef module = {PyModuleDef_HEAD_INIT, "_qmm_call", NULL, -1, methods,
                                    NULL, NULL, NULL, NULL};

PyMODINIT_FUNC PyInit__qmm_call(void) { return PyModule_Create(&module); }
