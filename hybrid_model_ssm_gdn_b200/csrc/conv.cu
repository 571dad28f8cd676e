// conv.cu -- in-house comparison kernels: conventional step-by-step decoding and
// snapshot-per-draft speculation.
//
// Conventional decoding loads the state, updates it, computes the output from the
// updated state and stores it back every token, so over a window of L tokens the state
// is read L times and written L times ("Hybrid-model decoding has a new bottleneck",
// Interpretation, second paragraph).  Snapshot speculation stores a state after every
// draft token and later picks the one matching the accepted prefix: one read and T
// writes per verification (same page, third paragraph).  Both are written here with the
// same memory discipline as the replay kernels (128-bit coalesced rows, streaming cache
// hints, warp transpose reductions) so that the comparison measures the scheme, not the
// code quality.  One block per (sequence, head); warp w owns rows ROWS*w.., lane l owns
// columns 4l..4l+3 of every row.
#include "kernels.h"

namespace rssm {

namespace {

template <int V>
__device__ __forceinline__ float row_sum_owner(float (&v)[V], int lane, int rr) {
  // after warp_transpose_reduce<V> with V <= 32, row rr lives in lane rr * (32 / V)
  return __shfl_sync(0xffffffffu, v[0], rr * (32 / V));
}

template <typename TI, int KIND, int ROWS>
__global__ void __launch_bounds__(256) conv_kernel(ConvArgs a) {
  const int unit = blockIdx.x;
  const int b = unit / a.H, h = unit % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = a.R;
  const size_t tile = (size_t)R * kCols;
  const int nslots = a.tmax + 1;
  float *src;
  if (a.cur) src = a.S + ((size_t)b * nslots + a.cur[b]) * a.H * tile + (size_t)h * tile;
  else src = a.S + (size_t)unit * tile;
  const int row0 = warp * ROWS;

  float4 s[ROWS];
#pragma unroll
  for (int rr = 0; rr < ROWS; ++rr)
    s[rr] = (row0 + rr < R) ? __ldcs(reinterpret_cast<const float4 *>(src + (row0 + rr) * kCols) + lane)
                            : make_float4(0, 0, 0, 0);

  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t)b * a.T + t;
    float part[ROWS];
    if (KIND == RSSM_MAMBA2) {
      const int g = h / (a.H / a.G);
      const float dt = to_f32(reinterpret_cast<const TI *>(a.dt)[tok * a.H + h]);
      const float dA = __expf(dt * a.A[h]);
      const TI *xp = reinterpret_cast<const TI *>(a.x) + (tok * a.H + h) * R;
      const float4 bv = load4(reinterpret_cast<const TI *>(a.Bin) + (tok * a.G + g) * kCols + 4 * lane);
      const float4 cv = load4(reinterpret_cast<const TI *>(a.C) + (tok * a.G + g) * kCols + 4 * lane);
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr) {
        const float cx = (row0 + rr < R) ? dt * to_f32(xp[row0 + rr]) : 0.f;
        s[rr].x = fmaf(dA, s[rr].x, cx * bv.x);
        s[rr].y = fmaf(dA, s[rr].y, cx * bv.y);
        s[rr].z = fmaf(dA, s[rr].z, cx * bv.z);
        s[rr].w = fmaf(dA, s[rr].w, cx * bv.w);
        part[rr] = s[rr].x * cv.x + s[rr].y * cv.y + s[rr].z * cv.z + s[rr].w * cv.w;
      }
      warp_transpose_reduce<ROWS>(part, lane);
      constexpr int SPREAD = 32 / ROWS;
      if (lane % SPREAD == 0) {
        const int p = row0 + lane / SPREAD;
        if (p < R) a.y[(tok * a.H + h) * R + p] = part[0] + a.D[h] * to_f32(xp[p]);
      }
    } else {
      const float al = a.alpha[tok * a.H + h], be = a.beta[tok * a.H + h];
      const float4 kv = load4(reinterpret_cast<const TI *>(a.k) + (tok * a.H + h) * kCols + 4 * lane);
      const float4 qv = load4(reinterpret_cast<const TI *>(a.q) + (tok * a.H + h) * kCols + 4 * lane);
      const TI *vp = reinterpret_cast<const TI *>(a.v) + (tok * a.H + h) * R;
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr) part[rr] = s[rr].x * kv.x + s[rr].y * kv.y + s[rr].z * kv.z + s[rr].w * kv.w;
      warp_transpose_reduce<ROWS>(part, lane);
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr) {
        const float sk = row_sum_owner<ROWS>(part, lane, rr);
        const float vr = (row0 + rr < R) ? to_f32(vp[row0 + rr]) : 0.f;
        const float coef = be * (vr - al * sk);  // S <- alpha S + beta (v - alpha S k) k^T
        s[rr].x = fmaf(al, s[rr].x, coef * kv.x);
        s[rr].y = fmaf(al, s[rr].y, coef * kv.y);
        s[rr].z = fmaf(al, s[rr].z, coef * kv.z);
        s[rr].w = fmaf(al, s[rr].w, coef * kv.w);
      }
      float yq[ROWS];
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr) yq[rr] = s[rr].x * qv.x + s[rr].y * qv.y + s[rr].z * qv.z + s[rr].w * qv.w;
      warp_transpose_reduce<ROWS>(yq, lane);
      constexpr int SPREAD = 32 / ROWS;
      if (lane % SPREAD == 0) {
        const int p = row0 + lane / SPREAD;
        if (p < R) a.y[(tok * a.H + h) * R + p] = a.q_scale * yq[0];
      }
    }
    if (a.cur) {  // snapshot after every draft token
      float *dst = a.S + ((size_t)b * nslots + (a.cur[b] + t + 1) % nslots) * a.H * tile + (size_t)h * tile;
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr)
        if (row0 + rr < R) __stcs(reinterpret_cast<float4 *>(dst + (row0 + rr) * kCols) + lane, s[rr]);
    }
  }
  if (!a.cur) {
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr)
      if (row0 + rr < R) __stcs(reinterpret_cast<float4 *>(src + (row0 + rr) * kCols) + lane, s[rr]);
  }
}

__global__ void snap_commit_kernel(int *cur, const int *accepted, int Bt, int nslots) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= Bt) return;
  int acc = accepted[b];
  acc = acc < 0 ? 0 : (acc >= nslots ? nslots - 1 : acc);
  cur[b] = (cur[b] + acc) % nslots;
}

}  // namespace

cudaError_t launch_conv(ConvArgs a, int esz, cudaStream_t stream) {
  const unsigned grid = (unsigned)(a.Bt * a.H);
  if (a.kind == RSSM_MAMBA2) {
    if (esz == 2) conv_kernel<__nv_bfloat16, RSSM_MAMBA2, 8><<<grid, 256, 0, stream>>>(a);
    else conv_kernel<float, RSSM_MAMBA2, 8><<<grid, 256, 0, stream>>>(a);
  } else {
    if (esz == 2) conv_kernel<__nv_bfloat16, RSSM_GDN, 16><<<grid, 256, 0, stream>>>(a);
    else conv_kernel<float, RSSM_GDN, 16><<<grid, 256, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_snap_commit(int *cur, const int *accepted, int Bt, int nslots, cudaStream_t stream) {
  snap_commit_kernel<<<(Bt + 255) / 256, 256, 0, stream>>>(cur, accepted, Bt, nslots);
  return cudaGetLastError();
}

}  // namespace rssm
