/*
 * _fastcall: a CPython extension that forwards one pre-marshalled
 * ragged_pipeline call, or one launch of a recorded pipeline graph
 * (ragged_pipeline_graph_launch), to the C ABI in a single Python -> C
 * crossing.
 *
 * The Python binding builds the argument block (struct pipeline_args, the
 * parameters of ragged_pipeline in order) once per buffer set and passes its
 * address; run() reads it and calls the ragged_pipeline function whose
 * address bind() received from the loaded libragged.  Argument marshalling
 * only: no computation happens here.  The GIL is released around the call,
 * which may block when RAGGED_PIPELINE_SYNC is set.
 */
#define PY_SSIZE_T_CLEAN
#include <Python.h>
#include <stdint.h>

typedef int (*pipeline_fn)(const void *, const uint8_t *, int64_t, int64_t, int64_t, int64_t, float, int,
                           void *, int32_t *, void *, void *, uint32_t, void *);

typedef struct {
    const void *dense_qkv;
    const uint8_t *keep;
    int64_t B, L_full, H, head_dim;
    float scale;
    int32_t dtype;
    void *packed_qkv;
    int32_t *cu_seqlens;
    void *out;
    void *cls_out;
    uint32_t flags;
    void *stream;
} pipeline_args;

static pipeline_fn g_pipeline = NULL;

typedef int (*graph_launch_fn)(void *, void *, uint32_t);

typedef struct {
    void *graph;
    void *stream;
    uint32_t flags;
} graph_args;

static graph_launch_fn g_graph_launch = NULL;

static PyObject *fc_bind(PyObject *self, PyObject *arg)
{
    (void)self;
    void *p = PyLong_AsVoidPtr(arg);
    if (p == NULL && PyErr_Occurred())
        return NULL;
    g_pipeline = (pipeline_fn)p;
    Py_RETURN_NONE;
}

static PyObject *fc_run(PyObject *self, PyObject *arg)
{
    (void)self;
    const pipeline_args *a = (const pipeline_args *)PyLong_AsVoidPtr(arg);
    if (a == NULL) {
        if (!PyErr_Occurred())
            PyErr_SetString(PyExc_ValueError, "null argument block");
        return NULL;
    }
    if (g_pipeline == NULL) {
        PyErr_SetString(PyExc_RuntimeError, "ragged_pipeline is not bound");
        return NULL;
    }
    int status;
    Py_BEGIN_ALLOW_THREADS
    status = g_pipeline(a->dense_qkv, a->keep, a->B, a->L_full, a->H, a->head_dim, a->scale, a->dtype,
                        a->packed_qkv, a->cu_seqlens, a->out, a->cls_out, a->flags, a->stream);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(status);
}

static PyObject *fc_bind_graph(PyObject *self, PyObject *arg)
{
    (void)self;
    void *p = PyLong_AsVoidPtr(arg);
    if (p == NULL && PyErr_Occurred())
        return NULL;
    g_graph_launch = (graph_launch_fn)p;
    Py_RETURN_NONE;
}

static PyObject *fc_graph_run(PyObject *self, PyObject *arg)
{
    (void)self;
    const graph_args *a = (const graph_args *)PyLong_AsVoidPtr(arg);
    if (a == NULL) {
        if (!PyErr_Occurred())
            PyErr_SetString(PyExc_ValueError, "null argument block");
        return NULL;
    }
    if (g_graph_launch == NULL) {
        PyErr_SetString(PyExc_RuntimeError, "ragged_pipeline_graph_launch is not bound");
        return NULL;
    }
    int status;
    Py_BEGIN_ALLOW_THREADS
    status = g_graph_launch(a->graph, a->stream, a->flags);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(status);
}

static PyObject *fc_graph_args_size(PyObject *self, PyObject *unused)
{
    (void)self;
    (void)unused;
    return PyLong_FromSize_t(sizeof(graph_args));
}

static PyObject *fc_args_size(PyObject *self, PyObject *unused)
{
    (void)self;
    (void)unused;
    return PyLong_FromSize_t(sizeof(pipeline_args));
}

static PyMethodDef fc_methods[] = {
    {"bind", fc_bind, METH_O, "bind(address of ragged_pipeline)"},
    {"run", fc_run, METH_O, "run(address of a pipeline argument block) -> ragged_status"},
    {"args_size", fc_args_size, METH_NOARGS, "size in bytes of the argument block"},
    {"bind_graph", fc_bind_graph, METH_O, "bind(address of ragged_pipeline_graph_launch)"},
    {"graph_run", fc_graph_run, METH_O, "graph_run(address of a graph argument block) -> ragged_status"},
    {"graph_args_size", fc_graph_args_size, METH_NOARGS, "size in bytes of the graph argument block"},
    {NULL, NULL, 0, NULL},
};

static struct PyModuleDef fc_module = {PyModuleDef_HEAD_INIT, "_fastcall",
                                       "Single-crossing forwarder for ragged_pipeline.", -1, fc_methods};

PyMODINIT_FUNC PyInit__fastcall(void) { return PyModule_Create(&fc_module); }
