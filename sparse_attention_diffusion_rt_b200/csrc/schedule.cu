// Denoising-schedule driver: which call step t of a calibration cycle makes,
// and one cycle captured as a CUDA graph.  The pages calibrate every few
// denoising steps ("Re-ttention": rho and the residual come from a periodic
// full-attention step and are reused, with the ramp-up lambda growing over the
// steps since, by the sparse steps in between).
#include <cuda_runtime.h>

#include <new>

#include "nvtx_range.h"
#include "rt.h"

namespace rtb {
rt_status api_cuda_fail(cudaError_t e, const char* where);
}

struct rt_cycle_graph {
  cudaGraphExec_t exec;
};

extern "C" {

rt_status rt_schedule_step(const rt_attn_desc* desc, const rt_schedule* sched, int32_t t, const void* q,
                           const void* k, const void* v, const rt_block_index* idx, void* o, float* rho, void* r,
                           void* stream) {
  RT_RANGE("rt_schedule_step");
  if (!sched || sched->period < 1 || t < 0) return RT_ERR_INVALID_ARGUMENT;
  const int32_t kdist = t % sched->period;
  if (kdist == 0) return rt_calibrate_ex(desc, q, k, v, idx, o, rho, r, sched->residual, stream);
  return rt_sparse_step_ex(desc, q, k, v, idx, rho, r, sched->lambda, kdist, sched->ramp, sched->epilogue, o,
                           stream);
}

rt_status rt_schedule_capture(const rt_attn_desc* desc, const rt_schedule* sched, const void* const* q,
                              const void* const* k, const void* const* v, const rt_block_index* idx,
                              void* const* o, float* rho, void* r, void* stream, rt_cycle_graph** graph) {
  RT_RANGE("rt_schedule_capture");
  if (!graph) return RT_ERR_INVALID_ARGUMENT;
  *graph = nullptr;
  if (!sched || sched->period < 1 || !q || !k || !v || !o || !stream) return RT_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamBeginCapture(s, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) return rtb::api_cuda_fail(e, "cudaStreamBeginCapture");
  rt_status st = RT_OK;
  for (int32_t t = 0; t < sched->period && st == RT_OK; ++t)
    st = rt_schedule_step(desc, sched, t, q[t], k[t], v[t], idx, o[t], rho, r, stream);
  cudaGraph_t g = nullptr;
  e = cudaStreamEndCapture(s, &g);
  if (st != RT_OK || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return st != RT_OK ? st : rtb::api_cuda_fail(e, "cudaStreamEndCapture");
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) return rtb::api_cuda_fail(e, "cudaGraphInstantiate");
  rt_cycle_graph* h = new (std::nothrow) rt_cycle_graph{exec};
  if (!h) {
    cudaGraphExecDestroy(exec);
    return RT_ERR_CUDA;
  }
  *graph = h;
  return RT_OK;
}

rt_status rt_cycle_graph_launch(rt_cycle_graph* graph, void* stream) {
  RT_RANGE("rt_cycle_graph_launch");
  if (!graph) return RT_ERR_INVALID_ARGUMENT;
  cudaError_t e = cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RT_OK : rtb::api_cuda_fail(e, "cudaGraphLaunch");
}

rt_status rt_cycle_graph_destroy(rt_cycle_graph* graph) {
  if (!graph) return RT_OK;
  cudaError_t e = cudaGraphExecDestroy(graph->exec);
  delete graph;
  return e == cudaSuccess ? RT_OK : rtb::api_cuda_fail(e, "cudaGraphExecDestroy");
}

}  // extern "C"
