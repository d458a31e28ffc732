// CPython entry points for the two calls a training or serving loop makes on
// every step, attn_fwd and attn_bwd. They only convert the Python ints and
// floats that the binding passes (data pointers, sizes, scale, stream handle)
// and call the library function whose address the binding hands in, so the
// library loaded by the binding is the one that runs. This is argument
// marshalling with less per-call interpreter work than a ctypes call; every
// check and all of the computation stay in the library.
//
// call_fwd(fn, q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, stream) -> int
// call_bwd(fn, q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes,
//          B, Hq, Hkv, N, d, scale, causal, stream) -> int
// Pointers and the stream are Python ints (None for null); the result is the
// library's status code. The GIL is released during the call, as ctypes does.
#define PY_SSIZE_T_CLEAN
#include <Python.h>
#include <limits.h>
#include <stddef.h>
#include <stdint.h>

typedef int (*fwd_fn)(const void*, const void*, const void*, void*, float*, int, int, int, int,
                      int, float, int, void*);
typedef int (*bwd_fn)(const void*, const void*, const void*, const void*, const float*,
                      const void*, void*, void*, void*, void*, size_t, int, int, int, int, int,
                      float, int, void*);

static int as_ptr(PyObject* o, void** out) {
  if (o == Py_None) {
    *out = NULL;
    return 0;
  }
  unsigned long long v = PyLong_AsUnsignedLongLong(o);
  if (v == (unsigned long long)-1 && PyErr_Occurred()) return -1;
  *out = (void*)(uintptr_t)v;
  return 0;
}

static int as_int(PyObject* o, int* out) {
  long v = PyLong_AsLong(o);
  if (v == -1 && PyErr_Occurred()) return -1;
  if (v < INT_MIN || v > INT_MAX) {
    PyErr_SetString(PyExc_OverflowError, "argument does not fit in a C int");
    return -1;
  }
  *out = (int)v;
  return 0;
}

static int as_float(PyObject* o, float* out) {
  double v = PyFloat_AsDouble(o);
  if (v == -1.0 && PyErr_Occurred()) return -1;
  *out = (float)v;
  return 0;
}

static int as_size(PyObject* o, size_t* out) {
  size_t v = PyLong_AsSize_t(o);
  if (v == (size_t)-1 && PyErr_Occurred()) return -1;
  *out = v;
  return 0;
}

static PyObject* call_fwd(PyObject* self, PyObject* const* args, Py_ssize_t n) {
  (void)self;
  if (n != 14) {
    PyErr_SetString(PyExc_TypeError, "call_fwd takes 14 arguments");
    return NULL;
  }
  void *fn, *p[5], *stream;
  int iv[5], causal;
  float scale;
  if (as_ptr(args[0], &fn)) return NULL;
  for (int i = 0; i < 5; ++i)
    if (as_ptr(args[1 + i], &p[i])) return NULL;
  for (int i = 0; i < 5; ++i)
    if (as_int(args[6 + i], &iv[i])) return NULL;
  if (as_float(args[11], &scale) || as_int(args[12], &causal) || as_ptr(args[13], &stream))
    return NULL;
  if (fn == NULL) {
    PyErr_SetString(PyExc_ValueError, "null function address");
    return NULL;
  }
  int st;
  Py_BEGIN_ALLOW_THREADS
  st = ((fwd_fn)fn)(p[0], p[1], p[2], p[3], (float*)p[4], iv[0], iv[1], iv[2], iv[3], iv[4],
                    scale, causal, stream);
  Py_END_ALLOW_THREADS
  return PyLong_FromLong(st);
}

static PyObject* call_bwd(PyObject* self, PyObject* const* args, Py_ssize_t n) {
  (void)self;
  if (n != 20) {
    PyErr_SetString(PyExc_TypeError, "call_bwd takes 20 arguments");
    return NULL;
  }
  void *fn, *p[10], *stream;
  size_t ws_bytes;
  int iv[5], causal;
  float scale;
  if (as_ptr(args[0], &fn)) return NULL;
  for (int i = 0; i < 10; ++i)
    if (as_ptr(args[1 + i], &p[i])) return NULL;
  if (as_size(args[11], &ws_bytes)) return NULL;
  for (int i = 0; i < 5; ++i)
    if (as_int(args[12 + i], &iv[i])) return NULL;
  if (as_float(args[17], &scale) || as_int(args[18], &causal) || as_ptr(args[19], &stream))
    return NULL;
  if (fn == NULL) {
    PyErr_SetString(PyExc_ValueError, "null function address");
    return NULL;
  }
  int st;
  Py_BEGIN_ALLOW_THREADS
  st = ((bwd_fn)fn)(p[0], p[1], p[2], p[3], (const float*)p[4], p[5], p[6], p[7], p[8], p[9],
                    ws_bytes, iv[0], iv[1], iv[2], iv[3], iv[4], scale, causal, stream);
  Py_END_ALLOW_THREADS
  return PyLong_FromLong(st);
}

static PyMethodDef kMethods[] = {
    {"call_fwd", (PyCFunction)(void (*)(void))call_fwd, METH_FASTCALL,
     "Call attn_fwd at the given address with converted arguments."},
    {"call_bwd", (PyCFunction)(void (*)(void))call_bwd, METH_FASTCALL,
     "Call attn_bwd at the given address with converted arguments."},
    {NULL, NULL, 0, NULL},
};

static struct PyModuleDef kModule = {
    PyModuleDef_HEAD_INIT, "_pycall", "Argument marshalling for attn_fwd and attn_bwd.", -1,
    kMethods, NULL, NULL, NULL, NULL,
};

PyMODINIT_FUNC PyInit__pycall(void) { return PyModule_Create(&kModule); }
