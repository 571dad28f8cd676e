// mamba2.cu -- ReplaySSM decode kernels for Mamba-2 layers (sm_100a).
//
// One persistent kernel serves decode steps, speculative verification and flushes.
// Per (sequence b, head h) the state is a fp32 checkpoint S0 in R^{P x 128} plus the
// inputs (x, B, dt) of the tokens since it, kept in a ring in HBM ("SSM decoding stops
// writing state every step", Synopsis and Interpretation, second paragraph).  For a
// call, the records of one unit are laid out as r = 0..n_rec-1 (buffered records in
// token order, then the call's new tokens); the first m of them are folded into the
// state and every output j replays records m..e_j-1 against the (possibly folded)
// state.  Unrolling the Mamba-2 recurrence S_t = exp(dt_t A) S_{t-1} + dt_t x_t B_t^T,
// y_t = S_t C_t + D x_t gives, with s(a, b) = sum_{a<=l<b} dt_l,
//
//   fold:   S' = exp(A s(0,m)) S0 + sum_{r<m} dt_r exp(A s(r+1,m)) x_r B_r^T
//   output: y_j = exp(A s(m,e_j)) S' C_j
//               + sum_{m<=r<e_j} dt_r exp(A s(r+1,e_j)) (B_r . C_j) x_r + D x_{e_j - 1}
//
// (the products of exp(dt A) are taken in log space).  Only a fold writes the state;
// a plain step reads the checkpoint once and writes its output and its input record.
//
// Data movement: a producer warp reads the bookkeeping word of the unit's sequence,
// decides the call's schedule (pre-fold / eager fold / error) and issues TMA bulk
// copies (cp.async.bulk, evict-first for the checkpoint stream) of the checkpoint tile,
// the buffered records and the new tokens into a shared-memory stage.  Eight consumer
// warps compute: warp w owns rows 8w..8w+7 of the tile, lane l owns columns 4l..4l+3,
// the row dot products with C are finished by a warp transpose reduction.
#include "common.cuh"
#include "kernels.h"

namespace rssm {

namespace {

// header ints / floats at the start of each stage
enum {
  H_FLAGS = 0,   // bit0 compute, bit1 state is written (m > 0), bit2 this unit writes the meta word
  H_NREC,        // records in the stage
  H_M,           // records folded into the state
  H_NRING,       // records taken from the ring (slots base_e + 0..n_ring-1)
  H_NNEW,        // new tokens of this call (appended)
  H_TOUT,        // outputs
  H_SLOT0,       // absolute ring slot of the first appended token
  H_MC, H_ME, H_MP,  // meta to write: count, epoch, pending
  H_B, H_H,
  H_BASE,        // absolute ring slot of buffered record 0 (window base before the call)
  H_F = 16       // floats from here: dt of new tokens [8], A, D
};
constexpr int kHdrBytes = 256;

struct M2Stage {
  int tile, xr, br, cr, dtr, bytes;
};

__host__ __device__ inline M2Stage m2_stage_layout(int P, int L, int tmax, int esz, int no) {
  M2Stage s;
  const int rmax = L + (tmax > 1 ? tmax : 1);
  s.tile = kHdrBytes;
  s.xr = s.tile + P * kCols * 4;
  s.br = (int)align_up(s.xr + rmax * P * esz, 16);
  s.cr = (int)align_up(s.br + rmax * kCols * esz, 16);
  s.dtr = (int)align_up(s.cr + no * kCols * esz, 16);
  s.bytes = (int)align_up(s.dtr + dt_stride(L) * 4, 128);
  return s;
}

constexpr int kTableFloats(int rmax, int no, int P) { return no * rmax + rmax + no + no * P; }

template <typename TI, int NO>
__global__ void __launch_bounds__(kThreads, 1) m2_replay_kernel(M2Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int esz = sizeof(TI);
  const M2Stage lay = m2_stage_layout(a.P, a.L, a.tmax, esz, NO);
  const int rmax = a.L + (a.tmax > 1 ? a.tmax : 1);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + a.nstage;
  float *tab = reinterpret_cast<float *>(smem + 16 * a.nstage);
  float *g_co = tab;                      // [NO][rmax] coefficient of record r in output j
  float *w_f = g_co + NO * rmax;          // [rmax]   fold weight of record r
  float *a_o = w_f + rmax;                // [NO]     checkpoint factor of output j
  float *extra = a_o + NO;                // [NO][P]  buffered part of output j
  float *a_f = extra + NO * a.P;          // [1]      checkpoint factor of the fold
  volatile int *abort_flag = reinterpret_cast<volatile int *>(a_f + 1);
  volatile int *issued = abort_flag + 1;    // units whose copies the producer has issued
  volatile int *consumed = abort_flag + 2;  // units the consumers have taken
  unsigned char *stages = smem + a.stage_base;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = (int)(((long long)blockIdx.x * a.units) / gridDim.x);
  const int u_end = (int)(((long long)(blockIdx.x + 1) * a.units) / gridDim.x);
  const int hpg = a.H / a.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    *issued = 0;
    *consumed = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------------ producer warp
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    int cached_b = -1;
    int4 meta = make_int4(0, 0, 0, 0);
    int msk = 1;
    for (int u = u_begin, i = 0; u < u_end; ++u, ++i) {
      const int s = i % a.nstage;
      const uint32_t ph = (uint32_t)((i / a.nstage) & 1);
      const int b = u / a.H, h = u % a.H, g = h / hpg;
      if (b != cached_b) {
        if (lane == 0) {
          meta = a.meta_in[b];
          msk = (a.mask == nullptr) ? 1 : (int)a.mask[b];
        }
        meta.x = __shfl_sync(0xffffffffu, meta.x, 0);
        meta.y = __shfl_sync(0xffffffffu, meta.y, 0);
        meta.z = __shfl_sync(0xffffffffu, meta.z, 0);
        msk = __shfl_sync(0xffffffffu, msk, 0);
        cached_b = b;
      }
      const int c = meta.x, e = meta.y, pend = meta.z;
      const int L = a.L;
      // ---- schedule of this unit (identical for every head of the sequence)
      int active = 1, n_ring = 0, n_new = 0, m = 0, t_out = 0, slot0 = 0;
      int mc = c, me = e, mp = pend;
      const int base_e = (e & 1) * L, base_n = ((e + 1) & 1) * L;
      if (pend != 0) {
        active = 0;
        if (h == 0 && lane == 0 && (a.op != OP_FLUSH || msk)) record_error(a.err, b, RSSM_DEV_PENDING);
      } else if (a.op == OP_STEP) {
        n_new = 1;
        t_out = 1;
        int c1;
        if (c == L) {  // pre-fold of a window completed by a commit
          n_ring = L; m = L; slot0 = base_n; c1 = 1; me = e + 1;
        } else {
          n_ring = c; m = 0; slot0 = base_e + c; c1 = c + 1;
        }
        if (c1 == L) { m = n_ring + 1; mc = 0; me = me + 1; }  // eager fold: the window is full
        else mc = c1;
      } else if (a.op == OP_VERIFY) {
        n_new = a.T;
        t_out = a.T;
        mp = a.T;
        if (c + a.T > L) { n_ring = c; m = c; slot0 = base_n; mc = 0; me = e + 1; }
        else { n_ring = c; m = 0; slot0 = base_e + c; }
      } else {  // flush
        if (!msk || c == 0) active = 0;
        else { n_ring = c; m = c; mc = 0; me = e + 1; }
      }
      const int n_rec = n_ring + n_new;
      if (!mbar_wait_or_abort(&empty[s], ph ^ 1u, abort_flag)) {
        if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      unsigned char *st = stages + (size_t)s * lay.bytes;
      int *hi = reinterpret_cast<int *>(st);
      float *hf = reinterpret_cast<float *>(st);
      if (lane == 0) {
        hi[H_FLAGS] = active | ((active && m > 0) ? 2 : 0) | (h == 0 ? 4 : 0);
        hi[H_NREC] = n_rec; hi[H_M] = m; hi[H_NRING] = n_ring; hi[H_NNEW] = n_new; hi[H_TOUT] = t_out;
        hi[H_SLOT0] = slot0; hi[H_MC] = mc; hi[H_ME] = me; hi[H_MP] = mp; hi[H_B] = b; hi[H_H] = h;
        hi[H_BASE] = base_e;
        hf[H_F + 8] = a.A[h];
        hf[H_F + 9] = a.D[h];
      }
      if (active && lane < n_new) {
        const TI *dtp = reinterpret_cast<const TI *>(a.dt) + ((size_t)b * a.T + lane) * a.H + h;
        hf[H_F + lane] = to_f32(*dtp);
      }
      __syncwarp();
      // ---- bulk copies
      uint32_t bytes = 0;
      const uint32_t tile_b = (uint32_t)a.P * kCols * 4;
      const uint32_t xrow = (uint32_t)a.P * esz, brow = (uint32_t)kCols * esz;
      if (active) bytes = tile_b + n_rec * (xrow + brow) + dt_stride(L) * 4 + t_out * brow;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes);
      __syncwarp();
      if (active) {
        const size_t unit = (size_t)b * a.H + h;
        // copy k is issued by lane k
        if (lane == 0) bulk_g2s(st + lay.tile, a.hp + unit * a.P * kCols, tile_b, &full[s], pol_stream);
        if (lane == 1 && n_ring)
          bulk_g2s(st + lay.xr, reinterpret_cast<const unsigned char *>(a.ring_x) + (unit * 2 * L + base_e) * xrow,
                   n_ring * xrow, &full[s], pol_keep);
        if (lane == 2 && n_ring)
          bulk_g2s(st + lay.br,
                   reinterpret_cast<const unsigned char *>(a.ring_B) + (((size_t)b * a.G + g) * 2 * L + base_e) * brow,
                   n_ring * brow, &full[s], pol_keep);
        if (lane == 3)
          bulk_g2s(st + lay.dtr, a.ring_dt + unit * dt_stride(L), dt_stride(L) * 4, &full[s], pol_keep);
        if (lane >= 4 && lane < 4 + n_new) {
          const int t = lane - 4;
          bulk_g2s(st + lay.xr + (n_ring + t) * xrow,
                   reinterpret_cast<const unsigned char *>(a.x) + (((size_t)b * a.T + t) * a.H + h) * xrow, xrow,
                   &full[s], pol_keep);
        }
        if (lane >= 12 && lane < 12 + n_new) {
          const int t = lane - 12;
          bulk_g2s(st + lay.br + (n_ring + t) * brow,
                   reinterpret_cast<const unsigned char *>(a.Bin) + (((size_t)b * a.T + t) * a.G + g) * brow, brow,
                   &full[s], pol_keep);
        }
        if (lane >= 20 && lane < 20 + t_out) {
          const int t = lane - 20;
          bulk_g2s(st + lay.cr + t * brow,
                   reinterpret_cast<const unsigned char *>(a.C) + (((size_t)b * a.T + t) * a.G + g) * brow, brow,
                   &full[s], pol_keep);
        }
      }
      if (lane == 0) *issued = i + 1;
    }
  } else {

  // -------------------------------------------------------------------- consumer warps
  const int tid = threadIdx.x;
  for (int u = u_begin, i = 0; u < u_end; ++u, ++i) {
    const int s = i % a.nstage;
    const uint32_t ph = (uint32_t)((i / a.nstage) & 1);
    if (!mbar_wait_or_abort(&full[s], ph, abort_flag) && lane == 0) {
      record_error(a.err, u / a.H, RSSM_DEV_TIMEOUT);
      *abort_flag = 1;
    }
    consumer_sync();  // a uniform decision: every consumer warp has waited (bounded) for this stage
    if (*abort_flag) break;
    if (tid == 0) *consumed = i + 1;
    const unsigned char *st = stages + (size_t)s * lay.bytes;
    const int *hi = reinterpret_cast<const int *>(st);
    const float *hf = reinterpret_cast<const float *>(st);
    const int flags = hi[H_FLAGS];
    const int b = hi[H_B], h = hi[H_H];
    if (flags & 4) {
      if (tid == 0) a.meta_out[b] = make_int4(hi[H_MC], hi[H_ME], hi[H_MP], 0);
    }
    if (flags & 1) {
      const int n_rec = hi[H_NREC], m = hi[H_M], n_ring = hi[H_NRING], n_new = hi[H_NNEW];
      const int t_out = hi[H_TOUT];
      const float A = hf[H_F + 8], Dh = hf[H_F + 9];
      const TI *xr = reinterpret_cast<const TI *>(st + lay.xr);
      const TI *br = reinterpret_cast<const TI *>(st + lay.br);
      const TI *cr = reinterpret_cast<const TI *>(st + lay.cr);
      const float *ring_dt = reinterpret_cast<const float *>(st + lay.dtr);
      const int base_e = hi[H_BASE];
      // dt of record r
      auto dt_of = [&](int r) -> float { return r < n_ring ? ring_dt[base_e + r] : hf[H_F + (r - n_ring)]; };
      // ---- P1: coefficients (pairs (j, r) with m <= r < e_j) and fold weights
      const int npairs = NO * n_rec;
      for (int pidx = warp; pidx < npairs; pidx += kConsumerWarps) {
        const int j = pidx / n_rec, r = pidx % n_rec;
        const int e_j = n_rec - t_out + j + 1;
        if (j >= t_out || r < m || r >= e_j) {
          if (lane == 0) g_co[j * rmax + r] = 0.f;
          continue;
        }
        const float4 bv = load4(br + r * kCols + 4 * lane);
        const float4 cv = load4(cr + j * kCols + 4 * lane);
        float d = bv.x * cv.x + bv.y * cv.y + bv.z * cv.z + bv.w * cv.w;
        d = warp_sum(d);
        if (lane == 0) {
          float sfx = 0.f;
          for (int l = r + 1; l < e_j; ++l) sfx += dt_of(l);
          g_co[j * rmax + r] = dt_of(r) * __expf(A * sfx) * d;
        }
      }
      if (tid < NO) {
        const int j = tid;
        if (j < t_out) {
          const int e_j = n_rec - t_out + j + 1;
          float sm = 0.f;
          for (int l = m; l < e_j; ++l) sm += dt_of(l);
          a_o[j] = __expf(A * sm);
        }
      }
      if (tid >= 64 && tid < 64 + m) {
        const int r = tid - 64;
        float sfx = 0.f;
        for (int l = r + 1; l < m; ++l) sfx += dt_of(l);
        w_f[r] = dt_of(r) * __expf(A * sfx);
      }
      if (tid == 128) {
        float sm = 0.f;
        for (int l = 0; l < m; ++l) sm += dt_of(l);
        *a_f = __expf(A * sm);
      }
      consumer_sync();
      // ---- P2: buffered part of each output row
      for (int q = tid; q < NO * a.P; q += kConsumers) {
        const int j = q / a.P, p = q % a.P;
        if (j >= t_out) break;
        const int e_j = n_rec - t_out + j + 1;
        float acc = Dh * to_f32(xr[(e_j - 1) * a.P + p]);
        for (int r = m; r < e_j; ++r) acc += g_co[j * rmax + r] * to_f32(xr[r * a.P + p]);
        extra[j * a.P + p] = acc;
      }
      consumer_sync();
      // ---- P3: stream the tile: fold (if any) and row dot products
      const float *tile = reinterpret_cast<const float *>(st + lay.tile);
      float4 cv[NO];
#pragma unroll
      for (int j = 0; j < NO; ++j) cv[j] = (j < t_out) ? load4(cr + j * kCols + 4 * lane) : make_float4(0, 0, 0, 0);
      const int row0 = warp * 8;
      if (row0 < a.P) {
        float4 sv[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) sv[rr] = *reinterpret_cast<const float4 *>(tile + (row0 + rr) * kCols + 4 * lane);
        if (m > 0) {
          const float af = *a_f;
#pragma unroll
          for (int rr = 0; rr < 8; ++rr) { sv[rr].x *= af; sv[rr].y *= af; sv[rr].z *= af; sv[rr].w *= af; }
          for (int r = 0; r < m; ++r) {
            const float4 bv = load4(br + r * kCols + 4 * lane);
            const float wr = w_f[r];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              const float cx = wr * to_f32(xr[r * a.P + row0 + rr]);
              sv[rr].x = fmaf(cx, bv.x, sv[rr].x);
              sv[rr].y = fmaf(cx, bv.y, sv[rr].y);
              sv[rr].z = fmaf(cx, bv.z, sv[rr].z);
              sv[rr].w = fmaf(cx, bv.w, sv[rr].w);
            }
          }
          float *dst = a.hp + ((size_t)b * a.H + h) * a.P * kCols;
#pragma unroll
          for (int rr = 0; rr < 8; ++rr) __stcs(reinterpret_cast<float4 *>(dst + (row0 + rr) * kCols + 4 * lane), sv[rr]);
        }
        float part[8 * NO];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
          for (int j = 0; j < NO; ++j)
            part[rr * NO + j] = sv[rr].x * cv[j].x + sv[rr].y * cv[j].y + sv[rr].z * cv[j].z + sv[rr].w * cv[j].w;
        warp_transpose_reduce<8 * NO>(part, lane);
        constexpr int V = 8 * NO;
        constexpr int KEEP = V >= 32 ? V / 32 : 1;
        constexpr int SPREAD = V >= 32 ? 1 : 32 / V;
        if ((lane % SPREAD) == 0) {
#pragma unroll
          for (int i2 = 0; i2 < KEEP; ++i2) {
            const int idx = (V >= 32) ? lane * KEEP + i2 : lane / SPREAD;
            const int rr = idx / NO, j = idx % NO;
            if (j < t_out) {
              const int p = row0 + rr;
              a.y[(((size_t)b * a.T + j) * a.H + h) * a.P + p] = a_o[j] * part[i2] + extra[j * a.P + p];
            }
          }
        }
      }
      // ---- P4: append the new tokens to the ring
      if (n_new) {
        const int slot0 = hi[H_SLOT0];
        const size_t unit = (size_t)b * a.H + h;
        const int xq = a.P * esz / 16;  // 16-byte chunks per x row
        for (int q = tid; q < n_new * xq; q += kConsumers) {
          const int t = q / xq, c16 = q % xq;
          const uint4 v = *reinterpret_cast<const uint4 *>(st + lay.xr + (n_ring + t) * a.P * esz + c16 * 16);
          *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(a.ring_x) +
                                     ((unit * 2 * a.L + slot0 + t) * a.P) * esz + c16 * 16) = v;
        }
        if (tid < n_new) a.ring_dt[unit * dt_stride(a.L) + slot0 + tid] = hf[H_F + tid];
        if (h % hpg == 0) {
          const int g = h / hpg;
          const int bq = kCols * esz / 16;
          for (int q = tid; q < n_new * bq; q += kConsumers) {
            const int t = q / bq, c16 = q % bq;
            const uint4 v = *reinterpret_cast<const uint4 *>(st + lay.br + (n_ring + t) * kCols * esz + c16 * 16);
            *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(a.ring_B) +
                                       ((((size_t)b * a.G + g) * 2 * a.L + slot0 + t) * kCols) * esz + c16 * 16) = v;
          }
        }
      }
    }
    // release the stage (all reads of it above are done) and the tables for the next unit
    consumer_sync();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // do not leave bulk copies in flight into shared memory of an exiting block
    for (int i = *consumed; i < *issued; ++i)
      if (!mbar_wait(&full[i % a.nstage], (uint32_t)((i / a.nstage) & 1))) break;
  }
}

}  // namespace

int m2_stage_bytes(int P, int L, int tmax, int esz, int no) { return m2_stage_layout(P, L, tmax, esz, no).bytes; }

int m2_table_bytes(int P, int L, int tmax, int no) {
  const int rmax = L + (tmax > 1 ? tmax : 1);
  return (int)align_up((size_t)(kTableFloats(rmax, no, P) + 4) * 4, 128);
}

cudaError_t launch_m2_replay(M2Args a, int esz, cudaStream_t stream) {
  const int no = a.tmax <= 1 ? 1 : a.tmax <= 2 ? 2 : a.tmax <= 4 ? 4 : 8;
  a.stage_base = (int)align_up(16 * a.nstage + m2_table_bytes(a.P, a.L, a.tmax, no), 128);
  const size_t smem = a.stage_base + (size_t)a.nstage * m2_stage_bytes(a.P, a.L, a.tmax, esz, no);
  void (*kern)(M2Args) = nullptr;
#define RSSM_PICK(TI, NOV) \
  if (no == NOV) kern = m2_replay_kernel<TI, NOV>;
  if (esz == 2) {
    RSSM_PICK(__nv_bfloat16, 1) RSSM_PICK(__nv_bfloat16, 2) RSSM_PICK(__nv_bfloat16, 4) RSSM_PICK(__nv_bfloat16, 8)
  } else {
    RSSM_PICK(float, 1) RSSM_PICK(float, 2) RSSM_PICK(float, 4) RSSM_PICK(float, 8)
  }
#undef RSSM_PICK
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<a.grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rssm
