// sched.cu -- self-test of the unit scheduler the replay kernels use, with no caller memory.
//
// The replay kernels hand (sequence, head-group) units to their persistent blocks through
// a counter in the context's arena (sched_grab / sched_finish in common.cuh): every unit
// goes to exactly one block, and the last block to finish re-arms the counter for the next
// launch on the stream.  rssm_sched_probe runs the same two helpers on counters, claim
// marks and per-block tallies held in file-scope device arrays, so a caller can check the
// mechanism on a device without allocating anything.  Calls must not overlap (one stream,
// or ordered streams): the arrays are shared by every caller of the library.
#include "sched.h"

namespace rssm {

namespace {

// [0] unused (the error-word slot of the arena layout), [1] next unit, [2] blocks finished
static __device__ int g_probe_sched[4];
static __device__ unsigned int g_probe_claims[kProbeMaxUnits];
static __device__ int g_probe_per_block[kProbeMaxBlocks];
static __device__ int g_probe_bad;

__global__ void probe_clear_kernel(int units) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x) g_probe_claims[u] = 0u;
  if (blockIdx.x == 0 && threadIdx.x == 0) g_probe_bad = 0;
}

// Each block draws units until the counter runs past `units`, marking every unit it draws.
__global__ void probe_draw_kernel(int units) {
  __shared__ int drawn_unit;
  int drawn = 0;
  for (;;) {
    if (threadIdx.x == 0) drawn_unit = sched_grab(g_probe_sched);
    __syncthreads();
    const int u = drawn_unit;
    __syncthreads();
    if (u >= units) break;
    if (threadIdx.x == 0) {
      atomicAdd(&g_probe_claims[u], 1u);
      ++drawn;
    }
  }
  if (threadIdx.x == 0) {
    g_probe_per_block[blockIdx.x] = drawn;
    sched_finish(g_probe_sched);
  }
}

// Counts units not drawn exactly once.
__global__ void probe_check_kernel(int units) {
  int bad = 0;
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x)
    bad += g_probe_claims[u] != 1u;
  if (bad) atomicAdd(&g_probe_bad, bad);
}

}  // namespace

cudaError_t launch_sched_probe(int units, int blocks, int *per_block, int *bad_units, cudaStream_t st) {
  probe_clear_kernel<<<64, 256, 0, st>>>(units);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    probe_draw_kernel<<<blocks, 32, 0, st>>>(units);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    probe_check_kernel<<<64, 256, 0, st>>>(units);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(per_block, g_probe_per_block, sizeof(int) * blocks, 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(bad_units, g_probe_bad, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e;
}

}  // namespace rssm
