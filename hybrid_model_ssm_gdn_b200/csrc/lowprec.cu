// lowprec.cu -- stand-alone precision converters: write a loaded fp32 checkpoint in the
// stored formats (fp32, fp16 or FP8 E4M3 with stochastic rounding at epoch 0, plus the
// NVFP4 read copy) and widen the stored checkpoint back to fp32 for export.  The rounding rules are
// those of lowprec.cuh.  One block of 64 threads per 64-row tile of a head's state;
// thread r owns row r (128 columns).
#include "kernels.h"
#include "lowprec.cuh"

namespace rssm {

namespace {

__global__ void store_state_kernel(const float *S, void *hp, float *hs, int hp_mode, unsigned char *rq,
                                   unsigned char *rs, float *rg, unsigned char *rc, int read_mode, int rows_per_head,
                                   unsigned long long seed) {
  const int nrb = (rows_per_head + kFp4Rows - 1) / kFp4Rows;
  const size_t unit = blockIdx.x / nrb;
  const int t = blockIdx.x % nrb;
  const int rows = min(kFp4Rows, rows_per_head - kFp4Rows * t);
  const int row = threadIdx.x;
  const bool live = row < rows;
  const int rowg = kFp4Rows * t + row;
  const float *src = S + (unit * rows_per_head + rowg) * kCols;
  __shared__ float red[64];
  float am = 0.f;
  if (live)
    for (int c = 0; c < kCols; ++c) am = fmaxf(am, fabsf(src[c]));
  // tile maximum (FP8 checkpoint scale, NVFP4 tile scale)
  red[row] = am;
  __syncthreads();
  float tmax = 0.f;
  for (int r = 0; r < kFp4Rows; ++r) tmax = fmaxf(tmax, red[r]);
  const bool fp8 = hp_mode == RSSM_HP_F8_SR && read_mode != RSSM_READ_SHARED_NVFP4;
  const float s8 = fp8_tile_scale(tmax);
  if (fp8 && row == 0) hs[unit * nrb + t] = s8;
  if (read_mode != RSSM_READ_SHARED_NVFP4 && live) {
    if (hp_mode == RSSM_HP_F8_SR) {
      unsigned char *dst = reinterpret_cast<unsigned char *>(hp) + (unit * rows_per_head + rowg) * kCols;
      for (int c = 0; c < kCols; c += 4) {
        const uint32_t elem = (uint32_t)(rowg * kCols + c);
        const uint4 rw = philox4x32_10(make_uint4((uint32_t)unit, 0u, elem >> 2, 0u), (uint32_t)seed,
                                       (uint32_t)(seed >> 32));
        dst[c] = (unsigned char)fp8_sr_code(__fdiv_rn(src[c], s8), rw.x);
        dst[c + 1] = (unsigned char)fp8_sr_code(__fdiv_rn(src[c + 1], s8), rw.y);
        dst[c + 2] = (unsigned char)fp8_sr_code(__fdiv_rn(src[c + 2], s8), rw.z);
        dst[c + 3] = (unsigned char)fp8_sr_code(__fdiv_rn(src[c + 3], s8), rw.w);
      }
    } else if (hp_mode == RSSM_HP_F32) {
      float *dst = reinterpret_cast<float *>(hp) + (unit * rows_per_head + rowg) * kCols;
      for (int c = 0; c < kCols; ++c) dst[c] = src[c];
    } else {
      __half *dst = reinterpret_cast<__half *>(hp) + (unit * rows_per_head + rowg) * kCols;
      for (int c = 0; c < kCols; c += 4) {
        const uint32_t elem = (uint32_t)(rowg * kCols + c);
        const uint4 rw = philox4x32_10(make_uint4((uint32_t)unit, 0u, elem >> 2, 0u), (uint32_t)seed,
                                       (uint32_t)(seed >> 32));
        dst[c] = fp16_sr(src[c], rw.x);
        dst[c + 1] = fp16_sr(src[c + 1], rw.y);
        dst[c + 2] = fp16_sr(src[c + 2], rw.z);
        dst[c + 3] = fp16_sr(src[c + 3], rw.w);
      }
    }
  }
  if (read_mode == RSSM_READ_SAME) return;
  const float g = nvfp4_tile_scale(tmax);
  if (row == 0) rg[unit * nrb + t] = g;
  if (read_mode == RSSM_READ_NVFP4D) {
    // column maxima per group of 16 rows, the column-group steps k, then NVFP4 blocks of x / k
    __shared__ unsigned int cmax[kFp4Rows / 16][kCols];
    __shared__ float kst[kFp4Rows / 16][kCols];
    for (int q = row; q < kFp4Rows / 16 * kCols; q += kFp4Rows) cmax[q / kCols][q % kCols] = 0u;
    __syncthreads();
    if (live)
      for (int c = 0; c < kCols; ++c) atomicMax(&cmax[row >> 4][c], __float_as_uint(fabsf(src[c])));
    __syncthreads();
    const int ngr = (rows_per_head + 15) / 16, ngr_t = (rows + 15) / 16;
    for (int q = row; q < ngr_t * kCols; q += kFp4Rows) {
      float k;
      const uint32_t code = nvfp4d_col_scale(__uint_as_float(cmax[q / kCols][q % kCols]), g, &k);
      kst[q / kCols][q % kCols] = k;
      rc[(unit * ngr + (size_t)t * (kFp4Rows / 16)) * kCols + q] = (unsigned char)code;
    }
    __syncthreads();
    if (!live) return;
    const float *kr = kst[row >> 4];
    for (int blk = 0; blk < kCols / 16; ++blk) {
      float xv[16], bam = 0.f;
      for (int c = 0; c < 16; ++c) {
        const float k = kr[blk * 16 + c];
        xv[c] = k > 0.f ? __fdiv_rn(src[blk * 16 + c], k) : 0.f;
        bam = fmaxf(bam, fabsf(xv[c]));
      }
      float d_b;
      rs[(unit * rows_per_head + rowg) * (kCols / 16) + blk] = (unsigned char)nvfp4d_block_scale(bam, &d_b);
      for (int c = 0; c < 16; c += 2) {
        const uint32_t lo = nvfp4_code(xv[c], d_b), hi = nvfp4_code(xv[c + 1], d_b);
        rq[(unit * rows_per_head + rowg) * (kCols / 2) + (blk * 16 + c) / 2] = (unsigned char)(lo | (hi << 4));
      }
    }
    return;
  }
  if (!live) return;
  for (int blk = 0; blk < kCols / 16; ++blk) {
    float bam = 0.f;
    for (int c = 0; c < 16; ++c) bam = fmaxf(bam, fabsf(src[blk * 16 + c]));
    float d_b;
    rs[(unit * rows_per_head + rowg) * (kCols / 16) + blk] = (unsigned char)nvfp4_block_scale(bam, g, &d_b);
    for (int c = 0; c < 16; c += 2) {
      const uint32_t lo = nvfp4_code(src[blk * 16 + c], d_b), hi = nvfp4_code(src[blk * 16 + c + 1], d_b);
      rq[(unit * rows_per_head + rowg) * (kCols / 2) + (blk * 16 + c) / 2] = (unsigned char)(lo | (hi << 4));
    }
  }
}

__global__ void widen_state_kernel(const void *hp, const float *hs, int hp_mode, const unsigned char *rq,
                                   const unsigned char *rs, const float *rg, int read_mode, float *out,
                                   int rows_per_head) {
  const int nrb = (rows_per_head + kFp4Rows - 1) / kFp4Rows;
  const size_t unit = blockIdx.x / nrb;
  const int t = blockIdx.x % nrb;
  const int rows = min(kFp4Rows, rows_per_head - kFp4Rows * t);
  const int row = threadIdx.x;
  if (row >= rows) return;
  const size_t r = unit * rows_per_head + kFp4Rows * t + row;
  float *dst = out + r * kCols;
  if (read_mode == RSSM_READ_SHARED_NVFP4) {
    const float g = rg[unit * nrb + t];
    for (int blk = 0; blk < kCols / 16; ++blk) {
      const float d_b = __fmul_rn(e4m3_value(rs[r * (kCols / 16) + blk]), g);
      for (int c = 0; c < 16; ++c) {
        const uint32_t byte = rq[r * (kCols / 2) + (blk * 16 + c) / 2];
        dst[blk * 16 + c] = nvfp4_value(((c & 1) ? (byte >> 4) : byte) & 15u, d_b);
      }
    }
  } else if (hp_mode == RSSM_HP_F16_SR) {
    const __half *src = reinterpret_cast<const __half *>(hp) + r * kCols;
    for (int c = 0; c < kCols; ++c) dst[c] = __half2float(src[c]);
  } else if (hp_mode == RSSM_HP_F8_SR) {
    const unsigned char *src = reinterpret_cast<const unsigned char *>(hp) + r * kCols;
    const float s8 = hs[unit * nrb + t];
    for (int c = 0; c < kCols; ++c) dst[c] = __fmul_rn(e4m3_signed_value(src[c]), s8);
  } else {
    const float *src = reinterpret_cast<const float *>(hp) + r * kCols;
    for (int c = 0; c < kCols; ++c) dst[c] = src[c];
  }
}

}  // namespace

cudaError_t launch_store_state(const float *S, void *hp, float *hs, int hp_mode, unsigned char *rq, unsigned char *rs,
                               float *rg, unsigned char *rc, int read_mode, int units, int rows, unsigned long long seed,
                               int /*H*/, cudaStream_t stream) {
  const int nrb = (rows + kFp4Rows - 1) / kFp4Rows;
  store_state_kernel<<<(unsigned)((size_t)units * nrb), kFp4Rows, 0, stream>>>(S, hp, hs, hp_mode, rq, rs, rg, rc,
                                                                                 read_mode, rows, seed);
  return cudaGetLastError();
}

cudaError_t launch_widen_state(const void *hp, const float *hs, int hp_mode, const unsigned char *rq,
                               const unsigned char *rs, const float *rg, int read_mode, float *out, int units, int rows,
                               cudaStream_t stream) {
  const int nrb = (rows + kFp4Rows - 1) / kFp4Rows;
  widen_state_kernel<<<(unsigned)((size_t)units * nrb), kFp4Rows, 0, stream>>>(hp, hs, hp_mode, rq, rs, rg, read_mode,
                                                                                 out, rows);
  return cudaGetLastError();
}

}  // namespace rssm
