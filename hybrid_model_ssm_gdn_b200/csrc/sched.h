// sched.h -- launch interface of the unit-scheduler self-test (sched.cu) for the host API.
#pragma once

#include "common.cuh"

namespace rssm {

constexpr int kProbeMaxUnits = 1 << 16;
constexpr int kProbeMaxBlocks = 1024;

// Runs the self-test on the library's file-scope scratch array; per_block and bad_units are host memory.
cudaError_t launch_sched_probe(int units, int blocks, int *per_block, int *bad_units, cudaStream_t stream);

}  // namespace rssm
