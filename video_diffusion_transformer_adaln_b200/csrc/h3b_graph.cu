// CUDA Graph capture of a multi-block pass, for replay without the per-kernel
// launch cost: the ten launches of every block are recorded once, with their
// tensor maps and arguments, and h3b_graph_launch replays the whole pass as a
// single graph launch.
//
// The captured pass is h3b_blocks_forward itself, so the graph computes exactly
// what the stream launches compute (same kernels, same arguments); only the
// host-side enqueue cost and the gaps between launches go away. The graph keeps
// the pointers it was captured with: x, c, the weights and the workspace must
// stay allocated and in place for as long as the graph is used.
#include <cuda_runtime.h>

#include <new>
#include <string>

#include "h3b.h"
#include "h3b_internal.h"

struct h3b_graph_s {
  cudaGraph_t graph;
  cudaGraphExec_t exec;
  int device;
  int launches;  // kernel nodes in the graph
};

namespace {

h3b_status graph_fail(cudaError_t e, const char* where) {
  h3b::set_error_detail(std::string(where) + ": " + cudaGetErrorString(e));
  return H3B_ERR_CUDA;
}

int count_kernel_nodes(cudaGraph_t g) {
  size_t n = 0;
  if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess || n == 0) return 0;
  cudaGraphNode_t* nodes = new (std::nothrow) cudaGraphNode_t[n];
  if (!nodes) return 0;
  int k = 0;
  if (cudaGraphGetNodes(g, nodes, &n) == cudaSuccess)
    for (size_t i = 0; i < n; ++i) {
      cudaGraphNodeType t;
      if (cudaGraphNodeGetType(nodes[i], &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++k;
    }
  delete[] nodes;
  return k;
}

}  // namespace

extern "C" h3b_status h3b_graph_capture_blocks(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks,
                                               const float* c, void* x, void* ws, size_t ws_bytes,
                                               h3b_graph* out) {
  if (!out) {
    h3b::set_error_detail("out is NULL");
    return H3B_ERR_ARG;
  }
  *out = nullptr;
  if (h3b::profiling_enabled()) {
    h3b::set_error_detail("profiling is on: its event records cannot be part of a graph");
    return H3B_ERR_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return graph_fail(e, "cudaGetDevice");
  cudaStream_t s = nullptr;
  if ((e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking)) != cudaSuccess)
    return graph_fail(e, "cudaStreamCreateWithFlags");
  if ((e = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal)) != cudaSuccess) {
    cudaStreamDestroy(s);
    return graph_fail(e, "cudaStreamBeginCapture");
  }
  // Validation runs on the host before anything is enqueued, as on the stream path.
  const h3b_status st = h3b_blocks_forward(dims, w, n_blocks, c, x, ws, ws_bytes, s);
  cudaGraph_t g = nullptr;
  e = cudaStreamEndCapture(s, &g);  // always leave capture mode
  cudaStreamDestroy(s);
  if (st != H3B_OK) {
    if (g) cudaGraphDestroy(g);
    return st;
  }
  if (e != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    return graph_fail(e != cudaSuccess ? e : cudaErrorStreamCaptureInvalidated, "cudaStreamEndCapture");
  }
  cudaGraphExec_t exec = nullptr;
  if ((e = cudaGraphInstantiate(&exec, g, 0)) != cudaSuccess) {
    cudaGraphDestroy(g);
    return graph_fail(e, "cudaGraphInstantiate");
  }
  h3b_graph_s* h = new (std::nothrow) h3b_graph_s{g, exec, dev, count_kernel_nodes(g)};
  if (!h) {
    cudaGraphExecDestroy(exec);
    cudaGraphDestroy(g);
    h3b::set_error_detail("out of host memory");
    return H3B_ERR_ARG;
  }
  *out = h;
  return H3B_OK;
}

extern "C" h3b_status h3b_graph_launch(h3b_graph g, h3b_stream stream) {
  if (!g) {
    h3b::set_error_detail("graph is NULL");
    return H3B_ERR_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return graph_fail(e, "cudaGetDevice");
  if (dev != g->device) {
    h3b::set_error_detail("the current device is not the device the graph was captured on");
    return H3B_ERR_ARG;
  }
  if ((e = cudaGraphLaunch(g->exec, stream)) != cudaSuccess) return graph_fail(e, "cudaGraphLaunch");
  return H3B_OK;
}

extern "C" int h3b_graph_kernel_count(h3b_graph g) { return g ? g->launches : 0; }

extern "C" void h3b_graph_destroy(h3b_graph g) {
  if (!g) return;
  cudaGraphExecDestroy(g->exec);
  cudaGraphDestroy(g->graph);
  delete g;
}
