// sched.cu -- self-test of the unit scheduler the replay kernels use, with no caller memory.
//
// The replay kernels hand (sequence, head-group) units to their persistent blocks through
// a counter in the context's arena (sched_grab / sched_finish in common.cuh): every unit
// goes to exactly one block, and the last block to finish re-arms the counter for the next
// launch on the stream.  rssm_sched_probe runs the same two helpers on a counter, claim
// marks and per-block tallies held in one file-scope device array, so that a caller which
// cannot allocate device memory (a host process that only holds a driver context, or code
// that runs where allocation is forbidden, such as inside a memory-pool-managed region)
// can still check the mechanism on its device.
//
// The array lives in the library's device image: every device that loads the library
// holds it until the process exits, and every call shares it, so calls must not overlap
// on the GPU (one stream, or streams ordered by the caller); overlapping calls race on the
// counter and the marks.  Host code never names the array as if it were a device address:
// the first call on a device looks its address up once with cudaGetSymbolAddress (with
// that device current) and passes it to the kernels, so that first call should come
// before any stream capture.
#include <mutex>

#include "sched.h"

namespace rssm {

namespace {

// Layout (ints): [0] unused (the arena's error-word slot), [1] next unit, [2] blocks finished,
// [3] units drawn twice or more / never (filled by the check), [4] 1 if the counter was not
// re-armed; per-block tallies from kPerBlockOff, claim marks from kClaimsOff.
constexpr int kPerBlockOff = 64;
constexpr int kClaimsOff = kPerBlockOff + kProbeMaxBlocks;
constexpr int kScratchInts = kClaimsOff + kProbeMaxUnits;
static __device__ __align__(256) int g_probe_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
int *g_addr[kMaxDevices];  // device address of g_probe_scratch, per device ordinal

// Clears the marks, the result words and the counter, so that a launch that never finished
// (for instance one cut short by an error) leaves nothing behind for the next probe.
__global__ void probe_clear_kernel(int *sc, int units) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x) sc[kClaimsOff + u] = 0;
  if (blockIdx.x == 0 && threadIdx.x < 8) sc[threadIdx.x] = 0;
}

// Each block draws units until the counter runs past `units`, marking every unit it draws.
__global__ void probe_draw_kernel(int *sc, int units) {
  __shared__ int drawn_unit;
  int drawn = 0;
  for (;;) {
    if (threadIdx.x == 0) drawn_unit = sched_grab(sc);
    __syncthreads();
    const int u = drawn_unit;
    __syncthreads();
    if (u >= units) break;
    if (threadIdx.x == 0) {
      atomicAdd(&sc[kClaimsOff + u], 1);
      ++drawn;
    }
  }
  if (threadIdx.x == 0) {
    sc[kPerBlockOff + blockIdx.x] = drawn;
    sched_finish(sc);
  }
}

// Counts units not drawn exactly once, and checks that the last block re-armed the counter.
__global__ void probe_check_kernel(int *sc, int units) {
  int bad = 0;
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x)
    bad += sc[kClaimsOff + u] != 1;
  if (bad) atomicAdd(&sc[3], bad);
  if (blockIdx.x == 0 && threadIdx.x == 0 && (sc[1] != 0 || sc[2] != 0)) sc[4] = 1;
}

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t scratch_address(int **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_probe_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<int *>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_sched_probe(int units, int blocks, int *per_block, int *bad_units, cudaStream_t st) {
  int *sc = nullptr;
  cudaError_t e = scratch_address(&sc);
  if (e != cudaSuccess) return e;
  probe_clear_kernel<<<64, 256, 0, st>>>(sc, units);
  e = cudaGetLastError();
  if (e == cudaSuccess) {
    probe_draw_kernel<<<blocks, 32, 0, st>>>(sc, units);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    probe_check_kernel<<<64, 256, 0, st>>>(sc, units);
    e = cudaGetLastError();
  }
  int words[2] = {0, 0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(per_block, sc + kPerBlockOff, sizeof(int) * blocks, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(words, sc + 3, sizeof(words), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) *bad_units = words[0] + words[1];
  return e;
}

}  // namespace rssm
