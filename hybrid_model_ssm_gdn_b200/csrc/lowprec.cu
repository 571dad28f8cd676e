// lowprec.cu -- precision converters (placeholder until the converters land).
#include "kernels.h"

namespace rssm {
cudaError_t launch_store_state(const float *, void *, int, unsigned char *, unsigned char *, float *, int, int, int,
                               unsigned long long, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_widen_state(const void *, int, const unsigned char *, const unsigned char *, const float *, int,
                               float *, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace rssm
