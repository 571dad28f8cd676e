// mamba2.cu -- ReplaySSM decode kernels for Mamba-2 layers (sm_100a).
//
// One persistent kernel serves decode steps, speculative verification and flushes.
// Per (sequence b, head h) the state is a fp32 checkpoint S0 in R^{P x 128} plus the
// inputs (x, B, dt) of the tokens since it, kept in a ring in HBM ("SSM decoding stops
// writing state every step", Synopsis and Interpretation, second paragraph).  For a
// call, the records of a sequence are laid out as r = 0..n_rec-1 (buffered records in
// token order, then the call's new tokens); the first m of them are folded into the
// state and output j replays records m..e_j-1 against the (possibly folded) state.
// Unrolling S_t = exp(dt_t A) S_{t-1} + dt_t x_t B_t^T, y_t = S_t C_t + D x_t gives,
// with s(a, b) = sum_{a<=l<b} dt_l,
//
//   fold:   S' = exp(A s(0,m)) S0 + sum_{r<m} dt_r exp(A s(r+1,m)) x_r B_r^T
//   output: y_j = exp(A s(m,e_j)) S' C_j
//               + sum_{m<=r<e_j} dt_r exp(A s(r+1,e_j)) (B_r . C_j) x_r + D x_{e_j - 1}
//
// (products of exp(dt A) taken in log space).  Only a fold writes the state; a plain
// step reads the checkpoint once and writes its output and its input record.
//
// Work unit: (sequence, group of <= 16 heads sharing B and C).  Warp roles in a block:
//  * producer warp: issues TMA bulk copies (cp.async.bulk; evict-first for the
//    checkpoint stream) into a double-buffered group buffer (B, C and dt rows of the
//    unit) and into a ring of tile stages (one head's checkpoint tile + its x records);
//  * prep warp: one unit ahead of the consumers, computes from the group buffer the
//    dot products B_r . C_j and every head's decay weights into double-buffered tables,
//    appends the group's B records and writes the sequence's bookkeeping word;
//  * eight consumer warps: warp w owns rows 8w..8w+7 of every tile, lane l columns
//    4l..4l+3; a warp waits on the stage's full barrier, computes its rows (fold, dot
//    products, transpose reduction, buffered part of y) and releases the stage on its
//    own.  No block-wide barrier sits on the streaming path, so one block per SM keeps
//    the checkpoint stream in flight while the next unit is being prepared.
#include "common.cuh"
#include "kernels.h"

namespace rssm {

namespace {

constexpr int kHG = 16;          // heads per unit (a group is split into chunks of <= 16)
constexpr int kGHdr = 1024;      // group header bytes

// group header: ints then floats
enum {
  G_ACTIVE = 0, G_NREC, G_M, G_NRING, G_NNEW, G_TOUT, G_SLOT0, G_MC, G_ME, G_MP, G_B, G_G, G_H0, G_NH,
  G_BASE, G_WMETA, G_WB,
  G_A = 32,                  // floats: A[16]
  G_D = G_A + kHG,           // D[16]
  G_DT = G_D + kHG           // dt of new tokens [8][16]
};

struct M2Layout {
  int rmax, no;
  int tile_bytes;            // P*128*4
  int xr;                    // offset of the x records in a tile stage
  int stage_bytes;
  int gb_B, gb_C, gb_dt, gb_bytes;  // group buffer
  int tab_bytes;
  int cx_bytes;              // fold scratch: per consumer warp, wf_r x_r[row] for its 8 rows
};

__host__ __device__ inline M2Layout m2_layout(int P, int L, int tmax, int esz) {
  M2Layout l;
  l.no = tmax <= 1 ? 1 : tmax <= 2 ? 2 : tmax <= 4 ? 4 : 8;
  l.rmax = L + (tmax > 1 ? tmax : 1);
  l.tile_bytes = P * kCols * 4;
  l.xr = l.tile_bytes;
  l.stage_bytes = (int)align_up((size_t)l.xr + (size_t)l.rmax * P * esz, 128);
  l.gb_B = kGHdr;
  l.gb_C = (int)align_up((size_t)l.gb_B + (size_t)l.rmax * kCols * esz, 16);
  l.gb_dt = (int)align_up((size_t)l.gb_C + (size_t)l.no * kCols * esz, 16);
  l.gb_bytes = (int)align_up((size_t)l.gb_dt + (size_t)kHG * dt_stride(L) * 4, 128);
  // tables: g[no][rmax], coef[kHG][no][rmax], ao[kHG][no], wf[kHG][rmax], af[kHG], flags[8]
  const int floats = l.no * l.rmax + kHG * l.no * l.rmax + kHG * l.no + kHG * l.rmax + kHG + 8;
  l.tab_bytes = (int)align_up((size_t)floats * 4, 128);
  l.cx_bytes = (int)align_up((size_t)kConsumerWarps * l.rmax * 8 * 4, 128);
  return l;
}

// barriers: full[8], empty[8], gfull[3], gempty[3], tfull[2], tempty[2]; then armed phases (ints)
constexpr int kBarBytes = 512;  // mbarriers (26 x 8 B) + armed phases + abort flag
constexpr int kGB = 3;  // group buffers: the producer loads a unit's group data one unit ahead
constexpr int kM2Threads = kConsumers + 64;  // + producer warp + prep warp
constexpr int kProducerWarp = kConsumerWarps, kPrepWarp = kConsumerWarps + 1;

template <typename TI, int NO>
__global__ void __launch_bounds__(kM2Threads, 1) m2_replay_kernel(M2Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int esz = sizeof(TI);
  const M2Layout lay = m2_layout(a.P, a.L, a.tmax, esz);
  const int NS = a.nstage;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + 8;
  uint64_t *gfull = empty + 8;    // [kGB] group data landed
  uint64_t *gempty = gfull + kGB; // [kGB] consumers done with a unit's group data
  uint64_t *tfull = gempty + kGB; // [2] tables ready
  uint64_t *tempty = tfull + 2;   // [2] consumers done with the tables
  volatile int *armed = reinterpret_cast<volatile int *>(tempty + 2);  // last armed phase of full[0..7], gfull[..]
  volatile int *abort_flag = armed + 8 + kGB;
  const int rmax = lay.rmax;
  unsigned char *tabs = smem + kBarBytes;  // two table buffers
  float *cx_scratch = reinterpret_cast<float *>(tabs + 2 * lay.tab_bytes);  // [8 warps][rmax][8 rows]
  unsigned char *gbuf = tabs + 2 * lay.tab_bytes + lay.cx_bytes;
  unsigned char *stages = gbuf + kGB * lay.gb_bytes;
  struct Tables {
    float *g, *coef, *ao, *wf, *af;
  };
  auto tables = [&](int which) {
    Tables t;
    t.g = reinterpret_cast<float *>(tabs + (size_t)which * lay.tab_bytes);  // [NO][rmax]   B_r . C_j
    t.coef = t.g + NO * rmax;                                                // [kHG][NO][rmax]
    t.ao = t.coef + kHG * NO * rmax;                                         // [kHG][NO]
    t.wf = t.ao + kHG * NO;                                                  // [kHG][rmax]
    t.af = t.wf + kHG * rmax;                                                // [kHG]
    return t;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hpg = a.H / a.G;
  const int chunks = (hpg + kHG - 1) / kHG;
  const int units = a.Bt * a.G * chunks;
  const int u_begin = (int)(((long long)blockIdx.x * units) / gridDim.x);
  const int u_end = (int)(((long long)(blockIdx.x + 1) * units) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int s = 0; s < kGB; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], kConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kConsumerWarps);
    }
    for (int s = 0; s < 8 + kGB; ++s) armed[s] = -1;
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    // ================================================================== producer warp
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    const uint32_t xrow = (uint32_t)a.P * esz, brow = (uint32_t)kCols * esz;
    const int L = a.L, dts = dt_stride(L);
    // bookkeeping words: lane q holds sequence (first + q) of the block's range, loaded up front
    // (and refreshed every 32 sequences) so the issue loop never waits on a global load
    const int b_first = u_begin / (a.G * chunks);
    int mw_base = -1;
    int4 mw = make_int4(0, 0, 0, 0);
    int mk = 1;
    struct Sched {
      int b, g, h0, nh, active, n_ring, n_new, m, t_out, slot0, base_e;
    };
    // schedule of unit u (identical for every head of the sequence); loads nothing but the
    // prefetched bookkeeping words
    auto schedule = [&](int u, Sched &S, int *hdr) {
      const int b = u / (a.G * chunks), g = (u / chunks) % a.G, ch = u % chunks;
      S.b = b; S.g = g; S.h0 = g * hpg + ch * kHG; S.nh = min(kHG, hpg - ch * kHG);
      const int base32 = b_first + ((b - b_first) & ~31);
      if (base32 != mw_base) {
        const int bq = base32 + lane;
        if (bq < a.Bt) {
          mw = a.meta_in[bq];
          mk = (a.mask == nullptr) ? 1 : (int)a.mask[bq];
        }
        mw_base = base32;
      }
      const int src = b - base32;
      const int c = __shfl_sync(0xffffffffu, mw.x, src), e = __shfl_sync(0xffffffffu, mw.y, src);
      const int pend = __shfl_sync(0xffffffffu, mw.z, src), msk = __shfl_sync(0xffffffffu, mk, src);
      int active = 1, n_ring = 0, n_new = 0, m = 0, t_out = 0, slot0 = 0;
      int mc = c, me = e, mp = pend;
      const int base_e = (e & 1) * L, base_n = ((e + 1) & 1) * L;
      if (pend != 0) {
        active = 0;
        if (S.h0 == 0 && lane == 0 && (a.op != OP_FLUSH || msk)) record_error(a.err, b, RSSM_DEV_PENDING);
      } else if (a.op == OP_STEP) {
        n_new = 1;
        t_out = 1;
        int c1;
        if (c == L) { n_ring = L; m = L; slot0 = base_n; c1 = 1; me = e + 1; }   // pre-fold after a commit
        else { n_ring = c; m = 0; slot0 = base_e + c; c1 = c + 1; }
        if (c1 == L) { m = n_ring + 1; mc = 0; me = me + 1; }                   // eager fold: window full
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
      S.active = active; S.n_ring = n_ring; S.n_new = n_new; S.m = m; S.t_out = t_out; S.slot0 = slot0;
      S.base_e = base_e;
      if (hdr != nullptr && lane == 0) {
        hdr[G_ACTIVE] = active; hdr[G_NREC] = n_ring + n_new; hdr[G_M] = m; hdr[G_NRING] = n_ring;
        hdr[G_NNEW] = n_new; hdr[G_TOUT] = t_out; hdr[G_SLOT0] = slot0; hdr[G_MC] = mc; hdr[G_ME] = me;
        hdr[G_MP] = mp; hdr[G_B] = b; hdr[G_G] = g; hdr[G_H0] = S.h0; hdr[G_NH] = S.nh; hdr[G_BASE] = base_e;
        hdr[G_WMETA] = (S.h0 == 0); hdr[G_WB] = (ch == 0);
      }
    };
    // group data of unit u into buffer u % kGB (B records, B and C of the new tokens, dt rows)
    auto issue_group = [&](int u, int gi) -> bool {
      const int gs = gi % kGB;
      if (!mbar_wait_or_abort(&gempty[gs], (uint32_t)(((gi / kGB) & 1) ^ 1), abort_flag)) return false;
      unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      Sched S;
      schedule(u, S, reinterpret_cast<int *>(gb));
      __syncwarp();
      const int n_rec = S.n_ring + S.n_new;
      const uint32_t gbytes = S.active ? (uint32_t)(n_rec * brow + S.t_out * brow + S.nh * dts * 4) : 0u;
      if (lane == 0) {
        armed[8 + gs] = gi / kGB;
        mbar_arrive_expect_tx(&gfull[gs], gbytes);
      }
      __syncwarp();
      if (S.active) {
        if (lane == 0 && S.n_ring)
          bulk_g2s(gb + lay.gb_B,
                   reinterpret_cast<const unsigned char *>(a.ring_B) + (((size_t)S.b * a.G + S.g) * 2 * L + S.base_e) * brow,
                   S.n_ring * brow, &gfull[gs], pol_keep);
        if (lane == 1)
          bulk_g2s(gb + lay.gb_dt, a.ring_dt + ((size_t)S.b * a.H + S.h0) * dts, S.nh * dts * 4, &gfull[gs], pol_keep);
        if (lane >= 4 && lane < 4 + S.n_new) {
          const int t = lane - 4;
          bulk_g2s(gb + lay.gb_B + (S.n_ring + t) * brow,
                   reinterpret_cast<const unsigned char *>(a.Bin) + (((size_t)S.b * a.T + t) * a.G + S.g) * brow, brow,
                   &gfull[gs], pol_keep);
        }
        if (lane >= 12 && lane < 12 + S.t_out) {
          const int t = lane - 12;
          bulk_g2s(gb + lay.gb_C + t * brow,
                   reinterpret_cast<const unsigned char *>(a.C) + (((size_t)S.b * a.T + t) * a.G + S.g) * brow, brow,
                   &gfull[gs], pol_keep);
        }
      }
      return true;
    };
    bool ok = true;
    if (u_begin < u_end) ok = issue_group(u_begin, 0);
    int ti = 0;
    for (int u = u_begin, gi = 0; ok && u < u_end; ++u, ++gi) {
      if (u + 1 < u_end && !issue_group(u + 1, gi + 1)) {
        ok = false;
        break;
      }
      Sched S;
      schedule(u, S, nullptr);
      if (!S.active) continue;
      const int n_rec = S.n_ring + S.n_new;
      const uint32_t tbytes = (uint32_t)lay.tile_bytes + n_rec * xrow;
      for (int i = 0; i < S.nh; ++i, ++ti) {
        const int s = ti % NS;
        if (!mbar_wait_or_abort(&empty[s], (uint32_t)(((ti / NS) & 1) ^ 1), abort_flag)) {
          ok = false;
          break;
        }
        unsigned char *st = stages + (size_t)s * lay.stage_bytes;
        const size_t unit = (size_t)S.b * a.H + S.h0 + i;
        if (lane == 0) {
          armed[s] = ti / NS;
          mbar_arrive_expect_tx(&full[s], tbytes);
        }
        __syncwarp();
        if (lane == 0) bulk_g2s(st, a.hp + unit * a.P * kCols, lay.tile_bytes, &full[s], pol_stream);
        if (lane == 1 && S.n_ring)
          bulk_g2s(st + lay.xr, reinterpret_cast<const unsigned char *>(a.ring_x) + (unit * 2 * L + S.base_e) * xrow,
                   S.n_ring * xrow, &full[s], pol_keep);
        if (lane >= 4 && lane < 4 + S.n_new) {
          const int t = lane - 4;
          bulk_g2s(st + lay.xr + (S.n_ring + t) * xrow,
                   reinterpret_cast<const unsigned char *>(a.x) + (((size_t)S.b * a.T + t) * a.H + S.h0 + i) * xrow, xrow,
                   &full[s], pol_keep);
        }
      }
    }
    if (!ok && lane == 0) {
      record_error(a.err, 0, RSSM_DEV_TIMEOUT);
      *abort_flag = 1;
    }
  } else if (warp == kPrepWarp) {
    // ================================================================== prep warp
    for (int u = u_begin, gi = 0; u < u_end; ++u, ++gi) {
      const int gs = gi % kGB, tsl = gi & 1;
      if (!mbar_wait_or_abort(&gfull[gs], (uint32_t)((gi / kGB) & 1), abort_flag) ||
          !mbar_wait_or_abort(&tempty[tsl], (uint32_t)(((gi >> 1) & 1) ^ 1), abort_flag)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      const unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      const float *gf = reinterpret_cast<const float *>(gb);
      const int b = gh[G_B], g = gh[G_G], nh = gh[G_NH], h0 = gh[G_H0];
      if (gh[G_WMETA] && lane == 0) a.meta_out[b] = make_int4(gh[G_MC], gh[G_ME], gh[G_MP], 0);
      // per-head parameters and the new tokens' dt (global loads, kept off the producer's path)
      float *gfw = reinterpret_cast<float *>(gbuf + (size_t)gs * lay.gb_bytes);
      {  // all loads issued before any is used (at most 8 tokens x 16 heads = 4 per lane)
        const int nq = gh[G_ACTIVE] ? gh[G_NNEW] * nh : 0;
        float dtv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int q = lane + 32 * k, t = q / max(nh, 1), i = q % max(nh, 1);
          dtv[k] = q < nq ? to_f32(reinterpret_cast<const TI *>(a.dt)[((size_t)b * a.T + t) * a.H + h0 + i]) : 0.f;
        }
        const float Av = lane < nh ? a.A[h0 + lane] : 0.f, Dv = lane < nh ? a.D[h0 + lane] : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int q = lane + 32 * k;
          if (q < nq) gfw[G_DT + (q / nh) * kHG + q % nh] = dtv[k];
        }
        if (lane < nh) {
          gfw[G_A + lane] = Av;
          gfw[G_D + lane] = Dv;
        }
      }
      __syncwarp();
      if (gh[G_ACTIVE]) {
        const Tables T = tables(tsl);
        const int n_rec = gh[G_NREC], m = gh[G_M], n_ring = gh[G_NRING], n_new = gh[G_NNEW], t_out = gh[G_TOUT];
        const int slot0 = gh[G_SLOT0], base_e = gh[G_BASE];
        const int dts = dt_stride(a.L);
        const TI *Bg = reinterpret_cast<const TI *>(gb + lay.gb_B);
        const TI *Cg = reinterpret_cast<const TI *>(gb + lay.gb_C);
        const float *dtg = reinterpret_cast<const float *>(gb + lay.gb_dt);
        auto dt_of = [&](int i, int r) -> float {
          return r < n_ring ? dtg[i * dts + base_e + r] : gf[G_DT + (r - n_ring) * kHG + i];
        };
        // g[j][r] = B_r . C_j, eight records per task
        const int rblocks = (n_rec + 7) / 8;
        for (int task = 0; task < t_out * rblocks; ++task) {
          const int j = task / rblocks, r0 = (task % rblocks) * 8;
          const float4 cv = load4(Cg + j * kCols + 4 * lane);
          float pd[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int r = r0 + q < n_rec ? r0 + q : n_rec - 1;
            const float4 bv = load4(Bg + r * kCols + 4 * lane);
            pd[q] = bv.x * cv.x + bv.y * cv.y + bv.z * cv.z + bv.w * cv.w;
          }
          warp_transpose_reduce<8>(pd, lane);
          if ((lane & 3) == 0 && r0 + (lane >> 2) < n_rec) T.g[j * rmax + r0 + (lane >> 2)] = pd[0];
        }
        // B records of the new tokens go to the group's ring row (first chunk only)
        if (gh[G_WB]) {
          const int bq = kCols * esz / 16;
          for (int q = lane; q < n_new * bq; q += 32) {
            const int t = q / bq, c16 = q % bq;
            const uint4 v = *reinterpret_cast<const uint4 *>(gb + lay.gb_B + (n_ring + t) * kCols * esz + c16 * 16);
            *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(a.ring_B) +
                                       ((((size_t)b * a.G + g) * 2 * a.L + slot0 + t) * kCols) * esz + c16 * 16) = v;
          }
        }
        // x rows of the new tokens go to each head's ring row, straight from the inputs: eight
        // 16-byte loads in flight per lane before the stores
        {
          const int xq = a.P * esz / 16, nq = n_new * nh * xq;
          for (int q0 = 0; q0 < nq; q0 += 256) {
            uint4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int q = q0 + k * 32 + lane;
              if (q < nq) {
                const int c16 = q % xq, ti2 = q / xq, t = ti2 / nh, i = ti2 % nh;
                v[k] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const unsigned char *>(a.x) +
                                                        (((size_t)b * a.T + t) * a.H + h0 + i) * a.P * esz + c16 * 16);
              }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int q = q0 + k * 32 + lane;
              if (q < nq) {
                const int c16 = q % xq, ti2 = q / xq, t = ti2 / nh, i = ti2 % nh;
                const size_t unit = (size_t)b * a.H + h0 + i;
                *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(a.ring_x) +
                                           ((unit * 2 * a.L + slot0 + t) * a.P) * esz + c16 * 16) = v[k];
              }
            }
          }
        }
        // dt of the new tokens goes to each head's ring row
        for (int q = lane; q < n_new * nh; q += 32) {
          const int t = q / nh, i = q % nh;
          a.ring_dt[((size_t)b * a.H + h0 + i) * dts + slot0 + t] = gf[G_DT + t * kHG + i];
        }
        __syncwarp();
        // per-head weights of every record in every output (log-space suffix sums of dt):
        // coef[r] = dt_r exp(A s(r+1, e_j)) (B_r . C_j) for m <= r < e_j, plus D on the output's
        // own token r = e_j - 1, and 0 elsewhere; ao = exp(A s(m, e_j)) scales S' C_j
        for (int pr = lane; pr < nh * t_out; pr += 32) {
          const int i = pr / t_out, j = pr % t_out;
          const float A = gf[G_A + i];
          const int e_j = n_rec - t_out + j + 1;
          float *co = T.coef + (i * NO + j) * rmax;
          for (int r = e_j; r < n_rec; ++r) co[r] = 0.f;
          float sfx = 0.f;
          for (int r = e_j - 1; r >= m; --r) {
            const float d = dt_of(i, r);
            co[r] = d * __expf(A * sfx) * T.g[j * rmax + r];
            sfx += d;
          }
          for (int r = 0; r < m; ++r) co[r] = 0.f;
          co[e_j - 1] += gf[G_D + i];
          T.ao[i * NO + j] = __expf(A * sfx);
        }
        if (m > 0 && lane < nh) {
          const int i = lane;
          const float A = gf[G_A + i];
          float sfx = 0.f;
          for (int r = m - 1; r >= 0; --r) {
            const float d = dt_of(i, r);
            T.wf[i * rmax + r] = d * __expf(A * sfx);
            sfx += d;
          }
          T.af[i] = __expf(A * sfx);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfull[tsl]);
    }
  } else {
    // ================================================================== consumer warps
    const int row0 = warp * 8;
    int ti = 0;
    for (int u = u_begin, gi = 0; u < u_end; ++u, ++gi) {
      const int gs = gi % kGB, tsl = gi & 1;
      if (!mbar_wait_or_abort(&tfull[tsl], (uint32_t)((gi >> 1) & 1), abort_flag)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      const unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      const int b = gh[G_B], h0 = gh[G_H0], nh = gh[G_NH];
      if (gh[G_ACTIVE]) {
        const Tables T = tables(tsl);
        const float *t_coef = T.coef, *t_ao = T.ao, *t_wf = T.wf, *t_af = T.af;
        const int n_rec = gh[G_NREC], m = gh[G_M], t_out = gh[G_TOUT];
        const TI *Bg = reinterpret_cast<const TI *>(gb + lay.gb_B);
        const TI *Cg = reinterpret_cast<const TI *>(gb + lay.gb_C);
        // ---- stream the heads' tiles; each warp works and releases on its own
        float4 cv[NO];
#pragma unroll
        for (int j = 0; j < NO; ++j) cv[j] = (j < t_out) ? load4(Cg + j * kCols + 4 * lane) : make_float4(0, 0, 0, 0);
        constexpr int V = 8 * NO;
        constexpr int KEEP = V >= 32 ? V / 32 : 1;
        constexpr int SPREAD = V >= 32 ? 1 : 32 / V;
        for (int i = 0; i < nh; ++i, ++ti) {
          const int s = ti % NS;
          if (!mbar_wait_or_abort(&full[s], (uint32_t)((ti / NS) & 1), abort_flag)) {
            if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
            break;
          }
          const unsigned char *st = stages + (size_t)s * lay.stage_bytes;
          const float *tile = reinterpret_cast<const float *>(st);
          const TI *xr = reinterpret_cast<const TI *>(st + lay.xr);
          const int h = h0 + i;
          const size_t unit = (size_t)b * a.H + h;
          if (row0 < a.P) {
            float4 sv[8];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) sv[rr] = *reinterpret_cast<const float4 *>(tile + (row0 + rr) * kCols + 4 * lane);
            if (m > 0) {
              const float af = t_af[i];
#pragma unroll
              for (int rr = 0; rr < 8; ++rr) { sv[rr].x *= af; sv[rr].y *= af; sv[rr].z *= af; sv[rr].w *= af; }
              // lane r forms wf_r x_r[row] for the warp's 8 rows in its warp's scratch rows
              float *cxw = cx_scratch + (size_t)warp * rmax * 8;
              for (int r = lane; r < m; r += 32) {
                float xv[8];
                load8(xr + r * a.P + row0, xv);
                const float wr = t_wf[i * rmax + r];
                *reinterpret_cast<float4 *>(cxw + r * 8) = make_float4(wr * xv[0], wr * xv[1], wr * xv[2], wr * xv[3]);
                *reinterpret_cast<float4 *>(cxw + r * 8 + 4) = make_float4(wr * xv[4], wr * xv[5], wr * xv[6], wr * xv[7]);
              }
              __syncwarp();
              for (int r = 0; r < m; ++r) {
                const float4 bv = load4(Bg + r * kCols + 4 * lane);
                const float4 c0 = *reinterpret_cast<const float4 *>(cxw + r * 8);
                const float4 c1 = *reinterpret_cast<const float4 *>(cxw + r * 8 + 4);
                const float cx[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                  sv[rr].x = fmaf(cx[rr], bv.x, sv[rr].x);
                  sv[rr].y = fmaf(cx[rr], bv.y, sv[rr].y);
                  sv[rr].z = fmaf(cx[rr], bv.z, sv[rr].z);
                  sv[rr].w = fmaf(cx[rr], bv.w, sv[rr].w);
                }
              }
              __syncwarp();
              float *dst = a.hp + unit * a.P * kCols;
#pragma unroll
              for (int rr = 0; rr < 8; ++rr)
                __stcs(reinterpret_cast<float4 *>(dst + (row0 + rr) * kCols + 4 * lane), sv[rr]);
            }
            // S'[row] . (ao_j C_j) over this lane's 4 columns, plus the buffered part: lane r
            // (< n_rec) adds coef_{j,r} x_r[row] for the warp's 8 rows (one 16-byte load of x_r)
            float part[V];
#pragma unroll
            for (int j = 0; j < NO; ++j) {
              const float ao = (j < t_out) ? t_ao[i * NO + j] : 0.f;
              const float4 c4 = make_float4(ao * cv[j].x, ao * cv[j].y, ao * cv[j].z, ao * cv[j].w);
#pragma unroll
              for (int rr = 0; rr < 8; ++rr)
                part[rr * NO + j] = sv[rr].x * c4.x + sv[rr].y * c4.y + sv[rr].z * c4.z + sv[rr].w * c4.w;
            }
            for (int r = lane; r < n_rec; r += 32) {
              float xv[8];
              load8(xr + r * a.P + row0, xv);
#pragma unroll
              for (int j = 0; j < NO; ++j) {
                const float co = (j < t_out) ? t_coef[(i * NO + j) * rmax + r] : 0.f;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) part[rr * NO + j] = fmaf(co, xv[rr], part[rr * NO + j]);
              }
            }
            warp_transpose_reduce<V>(part, lane);
#pragma unroll
            for (int k2 = 0; k2 < KEEP; ++k2) {
              const int idx = (V >= 32) ? lane * KEEP + k2 : lane / SPREAD;
              const int rr = idx / NO, j = idx % NO;
              if (j < t_out && (lane % SPREAD) == 0)
                a.y[(((size_t)b * a.T + j) * a.H + h) * a.P + row0 + rr] = part[k2];
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
      }
      if (*abort_flag) break;
      __syncwarp();
      if (lane == 0) {  // this warp is done with the unit's group buffer and tables
        mbar_arrive(&gempty[gs]);
        mbar_arrive(&tempty[tsl]);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // do not leave bulk copies in flight into the shared memory of an exiting block
    for (int s = 0; s < 8; ++s)
      if (armed[s] >= 0) mbar_wait(&full[s], (uint32_t)(armed[s] & 1));
    for (int s = 0; s < kGB; ++s)
      if (armed[8 + s] >= 0) mbar_wait(&gfull[s], (uint32_t)(armed[8 + s] & 1));
  }
}

}  // namespace

int m2_smem_bytes(int P, int L, int tmax, int esz, int nstage) {
  const M2Layout l = m2_layout(P, L, tmax, esz);
  return kBarBytes + 2 * l.tab_bytes + l.cx_bytes + kGB * l.gb_bytes + nstage * l.stage_bytes;
}

int m2_max_stages(int P, int L, int tmax, int esz, int smem_budget) {
  int n = 8;
  while (n > 2 && m2_smem_bytes(P, L, tmax, esz, n) > smem_budget) --n;
  return n;
}

int m2_units(int Bt, int H, int G) {
  const int hpg = H / G;
  return Bt * G * ((hpg + kHG - 1) / kHG);
}

cudaError_t launch_m2_replay(M2Args a, int esz, cudaStream_t stream) {
  const int no = a.tmax <= 1 ? 1 : a.tmax <= 2 ? 2 : a.tmax <= 4 ? 4 : 8;
  const size_t smem = m2_smem_bytes(a.P, a.L, a.tmax, esz, a.nstage);
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
  kern<<<a.grid, kM2Threads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rssm
