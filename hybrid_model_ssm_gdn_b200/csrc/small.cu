// small.cu -- bookkeeping kernels: meta reset, commit (a buffer-pointer move), exports.
//
// Commit advances the per-sequence record count by the accepted draft length and clears
// the pending verify; nothing else is touched ("Hybrid-model decoding has a new
// bottleneck", Interpretation, third paragraph: the accepted prefix is committed by
// advancing the buffer pointer).  The bookkeeping word of a sequence is int4 {count,
// epoch, pending, 0}; every call reads one copy and writes the other (ping-pong), so
// that no block ever reads a word another block of the same launch writes.
#include "kernels.h"

namespace rssm {

namespace {

__global__ void meta_reset_kernel(int4 *meta, int Bt, int *err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 2 * Bt) meta[i] = make_int4(0, 0, 0, 0);
  if (i == 0) {
    err[0] = kErrClean;
    err[1] = 0;  // unit scheduler: next unit, blocks finished
    err[2] = 0;
  }
}

__global__ void commit_kernel(const int4 *meta_in, int4 *meta_out, const int *accepted, int Bt, int *err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= Bt) return;
  const int4 m = meta_in[b];
  const int acc = accepted[b];
  int4 o = m;
  if (m.z == 0) {
    record_error(err, b, RSSM_DEV_NO_VERIFY);
  } else if (acc < 0 || acc > m.z) {
    record_error(err, b, RSSM_DEV_ACCEPTED);
  } else {
    o.x = m.x + acc;
    o.z = 0;
  }
  meta_out[b] = o;
}

__global__ void export_meta_kernel(const int4 *meta, int *out, int Bt, int L) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= Bt) return;
  const int4 m = meta[b];
  out[4 * b + 0] = m.x;
  out[4 * b + 1] = m.y;
  out[4 * b + 2] = m.z;
  out[4 * b + 3] = (m.y & 1) * L;
}

// out[(b*X + x)][s] = in[(b*X + x)][base_b + s], rows of slot_bytes (multiple of 4); a capped grid
// strides over the rows, so any row count the host API accepts fits one launch
__global__ void gather_window_kernel(const unsigned char *in, unsigned char *out, const int4 *meta, int Bt, int X,
                                     size_t in_group_bytes, int slot_bytes, int L, size_t rows) {
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {  // row = (b*X + x)*L + s
    const int s = (int)(row % L);
    const size_t grp = row / L;
    const int b = (int)(grp / X);
    const int base = (meta[b].y & 1) * L;
    const uint32_t *src = reinterpret_cast<const uint32_t *>(in + grp * in_group_bytes + (size_t)(base + s) * slot_bytes);
    uint32_t *dst = reinterpret_cast<uint32_t *>(out + row * slot_bytes);
    for (int w = threadIdx.x; w < slot_bytes / 4; w += blockDim.x) dst[w] = src[w];
  }
}

}  // namespace

cudaError_t launch_meta_reset(int4 *meta, int Bt, int *err, cudaStream_t stream) {
  meta_reset_kernel<<<(2 * Bt + 255) / 256, 256, 0, stream>>>(meta, Bt, err);
  return cudaGetLastError();
}

cudaError_t launch_commit(const int4 *meta_in, int4 *meta_out, const int *accepted, int Bt, int *err,
                          cudaStream_t stream) {
  commit_kernel<<<(Bt + 255) / 256, 256, 0, stream>>>(meta_in, meta_out, accepted, Bt, err);
  return cudaGetLastError();
}

cudaError_t launch_export_meta(const int4 *meta, int *out, int Bt, int L, cudaStream_t stream) {
  export_meta_kernel<<<(Bt + 255) / 256, 256, 0, stream>>>(meta, out, Bt, L);
  return cudaGetLastError();
}

cudaError_t launch_gather_window(const unsigned char *in, unsigned char *out, const int4 *meta, int Bt, int X,
                                 size_t in_group_bytes, int slot_bytes, int L, cudaStream_t stream) {
  const size_t rows = (size_t)Bt * X * L;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)(rows < (size_t)(1u << 20) ? rows : (size_t)(1u << 20));
  gather_window_kernel<<<grid, 64, 0, stream>>>(in, out, meta, Bt, X, in_group_bytes, slot_bytes, L, rows);
  return cudaGetLastError();
}

}  // namespace rssm
