// wq_graph.cu -- a decode step's chain of few-token matmuls as one CUDA graph.
//
// "Accelerating LLM inference with CUDA Graph and INT4 quantization" (cnblogs), part 2:
// the kernels of an inference step are captured in a CUDA graph once; each step only
// updates the arguments that change (the activation and output pointers) in the
// instantiated graph and launches it with one call, which removes the per-kernel launch
// cost that dominates microsecond-long decode GEMVs.
//
// The graph is captured from a private stream: node i is the launch of the few-token matmul
// kernel of ops[i] with exactly the launch plan w4a16_gemm would use, made with programmatic
// dependent launch allowed, so the capture joins consecutive nodes with programmatic edges and
// node i+1 streams its weights while node i finishes.  Each node's handle is read from the
// capture right after its launch; wq_graph_set_io rebuilds one node's arguments for new
// pointers and writes them into the instantiated graph with cudaGraphExecKernelNodeSetParams.
#include <cuda_runtime.h>

#include <new>
#include <vector>

#include "wq_host.h"

struct wq_graph {
    std::vector<wq_matmul_desc> ops;
    std::vector<cudaGraphNode_t> nodes;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int device = -1;
};

namespace wq {
namespace {

wq_status prepare_op(const wq_matmul_desc &d, PreparedLaunch *L)
{
    wq_status rc = check_a16(d.A, d.a_dt, d.Wq, d.scales, d.zeros, d.bias, d.C, d.M, d.N, d.K, d.c);
    if (rc != WQ_OK) return rc;
    if (d.M > 16) return fail(WQ_ERR_UNSUPPORTED, "wq_graph: matmuls of at most 16 tokens (M=%lld)", (long long)d.M);
    const int am = d.a_dt == WQ_F16 ? 0 : 1;
    const int wf = wf_of(d.c);
    return gemv_prepare(wf, am, d.A, nullptr, d.Wq, d.scales, wf == WF_I4 && !d.c.symmetric ? d.zeros : nullptr,
                        d.bias, d.C, nullptr, d.M, d.N, d.K, d.c, L);
}

void release(wq_graph *g)
{
    if (!g) return;
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    delete g;
}

}  // namespace
}  // namespace wq

using namespace wq;

extern "C" wq_status wq_graph_create(const wq_matmul_desc *ops, int n_ops, wq_graph **out)
{
    if (!out) return fail(WQ_ERR_INVALID_ARG, "wq_graph_create: out must be non-null");
    *out = nullptr;
    if (!ops || n_ops < 1 || n_ops > WQ_GRAPH_MAX_OPS)
        return fail(WQ_ERR_INVALID_ARG, "wq_graph_create: 1 to %d matmuls", WQ_GRAPH_MAX_OPS);
    std::vector<PreparedLaunch> L(n_ops);
    for (int i = 0; i < n_ops; ++i) {
        const wq_status rc = prepare_op(ops[i], &L[i]);
        if (rc != WQ_OK) return rc;
    }
    wq_graph *g = new (std::nothrow) wq_graph;
    if (!g) return fail(WQ_ERR_INVALID_ARG, "wq_graph_create: out of host memory");
    g->ops.assign(ops, ops + n_ops);
    g->nodes.resize(n_ops);
    cudaGetDevice(&g->device);
    cudaStream_t cs = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
    bool capturing = e == cudaSuccess;
    wq_status rc = WQ_OK;
    for (int i = 0; i < n_ops && e == cudaSuccess; ++i) {
        rc = launch_prepared(L[i], cs, "wq_graph_create");
        if (rc != WQ_OK) break;
        cudaStreamCaptureStatus st;
        const cudaGraphNode_t *deps = nullptr;
        size_t nd = 0;
        e = cudaStreamGetCaptureInfo(cs, &st, nullptr, nullptr, &deps, &nd);
        if (e == cudaSuccess && (st != cudaStreamCaptureStatusActive || nd != 1)) e = cudaErrorStreamCaptureInvalidated;
        if (e == cudaSuccess) g->nodes[i] = deps[0];  // the node this launch added
    }
    if (capturing) {
        cudaGraph_t graph = nullptr;
        const cudaError_t e2 = cudaStreamEndCapture(cs, &graph);
        g->graph = graph;
        if (e == cudaSuccess) e = e2;
    }
    if (cs) cudaStreamDestroy(cs);
    if (rc == WQ_OK && e == cudaSuccess) e = cudaGraphInstantiate(&g->exec, g->graph, 0);
    if (rc != WQ_OK || e != cudaSuccess) {
        release(g);
        return rc != WQ_OK ? rc : fail(WQ_ERR_CUDA, "wq_graph_create: %s", cudaGetErrorString(e));
    }
    *out = g;
    return WQ_OK;
}

extern "C" wq_status wq_graph_set_io(wq_graph *g, int op, const void *A, void *C)
{
    if (!g) return fail(WQ_ERR_INVALID_ARG, "wq_graph_set_io: null graph");
    if (op < 0 || op >= int(g->ops.size())) return fail(WQ_ERR_INVALID_ARG, "wq_graph_set_io: op %d out of range", op);
    wq_matmul_desc d = g->ops[op];
    d.A = A;
    d.C = C;
    PreparedLaunch L;
    const wq_status rc = prepare_op(d, &L);
    if (rc != WQ_OK) return rc;
    const cudaKernelNodeParams kp = L.node_params();
    const cudaError_t e = cudaGraphExecKernelNodeSetParams(g->exec, g->nodes[op], &kp);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_graph_set_io: %s", cudaGetErrorString(e));
    g->ops[op] = d;
    return WQ_OK;
}

extern "C" wq_status wq_graph_launch(wq_graph *g, cudaStream_t stream)
{
    if (!g) return fail(WQ_ERR_INVALID_ARG, "wq_graph_launch: null graph");
    const cudaError_t e = cudaGraphLaunch(g->exec, stream);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_graph_launch: %s", cudaGetErrorString(e));
    return WQ_OK;
}

extern "C" void wq_graph_destroy(wq_graph *g) { release(g); }
