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
// Work unit: (sequence, group of <= 16 heads sharing B and C).  The persistent blocks draw
// units from a per-launch counter.  Warp roles in a block:
//  * producer warp: takes the next unit, writes its schedule into one of three group
//    buffers and issues TMA bulk copies (cp.async.bulk; evict-first for the checkpoint
//    stream) of the unit's B, C and dt rows into it, one unit ahead, then of each head's
//    checkpoint tile and x records into a ring of tile stages;
//  * prep warp: one unit ahead of the consumers, computes from the group buffer the
//    dot products B_r . C_j and every head's decay weights into double-buffered tables,
//    appends the group's B and dt records and writes the sequence's bookkeeping word;
//  * eight consumer warps: warp w owns rows 8w..8w+7 of every tile, lane l columns
//    4l..4l+3; a warp waits on the stage's full barrier, computes its rows (fold, dot
//    products, transpose reduction, buffered part of y), appends the head's new x rows
//    with one bulk store when it is its turn, and releases the stage on its own.  With
//    bf16 inputs and 5..8 outputs, S'.C and the buffered term run on tensor cores
//    (mma.sync, register operands).  With bf16 inputs, one output and windows up to 16, a
//    fold tile is taken by one group of four consumer warps (the groups alternate), each
//    warp owning 16 rows: S' = af S + X' B on tensor cores, X' = wf_r x_r cut into three
//    bf16 pieces whose sum is exact, B the group's records reordered by the prep warp for
//    ldmatrix.trans.  No block-wide barrier sits on the streaming path, so one block per SM
//    keeps the checkpoint stream in flight while the next unit is being prepared.
#include "common.cuh"
#include "kernels.h"

namespace rssm {

namespace {

constexpr int kHG = 16;          // heads per unit (a group is split into chunks of <= 16)
constexpr int kGHdr = 1024;      // group header bytes

// group header: ints then floats
enum {
  G_ACTIVE = 0, G_NREC, G_M, G_NRING, G_NNEW, G_TOUT, G_SLOT0, G_MC, G_ME, G_MP, G_B, G_G, G_H0, G_NH,
  G_BASE, G_WMETA, G_WB, G_SKIP, G_END,  // G_SKIP: bit i set = head h0 + i skips its checkpoint read
  G_A = 32,                  // floats: A[16]
  G_D = G_A + kHG,           // D[16]
  G_DT = G_D + kHG           // dt of new tokens [8][16]
};

constexpr int kBkPitch = 272;  // bytes per reordered B record (128 bf16 + 16)

struct M2Layout {
  int rmax, no;
  bool mma;                  // output contraction on tensor cores (bf16 inputs, 8 outputs per row)
  int nq;                    // 16-record steps of the buffered term on that path
  int tile_bytes;            // P*128*4
  int xr;                    // offset of the x records in a tile stage
  int stage_bytes;
  int gb_B, gb_C, gb_dt, gb_bytes;  // group buffer
  int tab_bytes;
  int tb_bk;                 // chunked fold: the folded B records, reordered, in each table buffer (0: none)
  int cx_bytes;              // fold scratch: per consumer warp, wf_r x_r[row] for its 8 rows
};

__host__ __device__ inline M2Layout m2_layout(int P, int L, int tmax, int esz) {
  M2Layout l;
  l.no = tmax <= 1 ? 1 : tmax <= 2 ? 2 : tmax <= 4 ? 4 : 8;
  l.mma = l.no == 8 && esz == 2;
  l.rmax = L + (tmax > 1 ? tmax : 1);
  l.nq = (l.rmax + 15) / 16;
  l.tile_bytes = P * kCols * 4;
  l.xr = l.tile_bytes;
  l.stage_bytes = (int)align_up((size_t)l.xr + (size_t)l.rmax * P * esz, 128);
  l.gb_B = kGHdr;
  l.gb_C = (int)align_up((size_t)l.gb_B + (size_t)l.rmax * kCols * esz, 16);
  l.gb_dt = (int)align_up((size_t)l.gb_C + (size_t)l.no * kCols * esz, 16);
  l.gb_bytes = (int)align_up((size_t)l.gb_dt + (size_t)kHG * dt_stride(L) * 4, 128);
  // tables: g[no][rmax], coef[kHG][no][rmax] (or, on the tensor-core path, its fragments
  // [kHG][nq][32 lanes][4 words]), ao[kHG][no], wf[kHG][rmax], af[kHG], flags[8]
  const int coef_floats = l.mma ? kHG * l.nq * 32 * 4 : kHG * l.no * l.rmax;
  const int floats = l.no * l.rmax + coef_floats + kHG * l.no + kHG * l.rmax + kHG + 8;
  // chunked fold (bf16 inputs, CUDA-core output path, windows up to 16): the folded B records, reordered for
  // ldmatrix.trans at a pitch of 272 bytes (no bank conflicts), in each table buffer
  const bool tcf = esz == 2 && (l.no == 1 || l.mma) && L <= 16;
  const size_t tb = align_up((size_t)floats * 4, 16);
  l.tb_bk = tcf ? (int)tb : 0;
  l.tab_bytes = (int)align_up(tb + (tcf ? (size_t)16 * kBkPitch : 0), 128);
  l.cx_bytes = (int)align_up((size_t)kConsumerWarps * l.rmax * 8 * 4, 128);
  return l;
}

// barriers: full[8], empty[8], gfull[3], gempty[3], tfull[2], tempty[2]; then armed phases (ints)
constexpr int kBarBytes = 512;  // mbarriers (26 x 8 B) + armed phases + abort flag
constexpr int kGB = 3;  // group buffers: the producer loads a unit's group data one unit ahead
constexpr int kM2Threads = kConsumers + 64;  // + producer warp + prep warp
constexpr int kProducerWarp = kConsumerWarps, kPrepWarp = kConsumerWarps + 1;

// TCF: the instance with the chunked fold on tensor cores (bf16 inputs, one output, windows up to 16).  Launches
// the host knows to be fold-free take the instance without it: its streaming path compiles as it did before the
// chunked fold (plain launches measured 5% slower with the fold code present, whether inline or out of line, and
// with the register allocation capped).  Both instances fold correctly; the choice only affects speed.
template <typename TI, int NO, bool TCF>
__global__ void __launch_bounds__(kM2Threads, 1) m2_replay_kernel(M2Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // S'.C_j on tensor cores for 5..8 drafts (measured: at 4 the CUDA-core reduction is as fast): C_j is
  // exact in bf16 and S' enters as a hi + lo bf16 pair
  constexpr bool kMma = NO == 8 && sizeof(TI) == 2;
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
    t.ao = t.coef + (kMma ? kHG * lay.nq * 32 * 4 : kHG * NO * rmax);       // [kHG][NO]
    t.wf = t.ao + kHG * NO;                                                  // [kHG][rmax]
    t.af = t.wf + kHG * rmax;                                                // [kHG]
    return t;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitSpec ws{a.wait_cycles, a.suspend_ns};
  const int hpg = a.H / a.G;
  const int chunks = (hpg + kHG - 1) / kHG;
  const int units = a.Bt * a.G * chunks;

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
    struct Sched {
      int b, g, h0, nh, active, n_ring, n_new, m, t_out, slot0, base_e;
      unsigned skip;
    };
    // schedule of unit u (identical for every head of the sequence) from the sequence's
    // bookkeeping word; u >= units writes the end marker
    auto schedule = [&](int u, Sched &S, int *hdr) {
      if (u >= units) {
        S = Sched{};
        if (lane == 0) { hdr[G_ACTIVE] = 0; hdr[G_END] = 1; }
        return;
      }
      const int b = u / (a.G * chunks), g = (u / chunks) % a.G, ch = u % chunks;
      S.b = b; S.g = g; S.h0 = g * hpg + ch * kHG; S.nh = min(kHG, hpg - ch * kHG);
      int4 mw = make_int4(0, 0, 0, 0);
      int mk = 1, fl = 0;
      if (lane == 0) {
        mw = a.meta_in[b];
        mk = (a.mask == nullptr) ? 1 : (int)a.mask[b];
      }
      // skip flags left by the previous call, loaded beside the bookkeeping word
      if (a.skip != nullptr && lane < S.nh) fl = a.skip[(size_t)b * a.H + S.h0 + lane];
      const unsigned skm = __ballot_sync(0xffffffffu, fl != 0);
      const int c = __shfl_sync(0xffffffffu, mw.x, 0), e = __shfl_sync(0xffffffffu, mw.y, 0);
      const int pend = __shfl_sync(0xffffffffu, mw.z, 0), msk = __shfl_sync(0xffffffffu, mk, 0);
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
      S.skip = active ? skm : 0u;
      if (lane == 0) {
        hdr[G_ACTIVE] = active; hdr[G_NREC] = n_ring + n_new; hdr[G_M] = m; hdr[G_NRING] = n_ring;
        hdr[G_NNEW] = n_new; hdr[G_TOUT] = t_out; hdr[G_SLOT0] = slot0; hdr[G_MC] = mc; hdr[G_ME] = me;
        hdr[G_MP] = mp; hdr[G_B] = b; hdr[G_G] = g; hdr[G_H0] = S.h0; hdr[G_NH] = S.nh; hdr[G_BASE] = base_e;
        hdr[G_WMETA] = (S.h0 == 0); hdr[G_WB] = (ch == 0); hdr[G_SKIP] = (int)S.skip; hdr[G_END] = 0;
      }
    };
    // group data of unit u into buffer gi % kGB (B records, B and C of the new tokens, dt rows)
    auto issue_group = [&](int u, int gi, Sched &S) -> bool {
      const int gs = gi % kGB;
      if (!mbar_wait_or_abort(&gempty[gs], (uint32_t)(((gi / kGB) & 1) ^ 1), abort_flag, ws)) return false;
      unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
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
    // units come from the launch's counter: the group data of the next unit is issued before
    // the current unit's tiles, and the unit after that is requested (atomic in flight) meanwhile
    int u_cur = 0, u_nxt = 0;
    if (lane == 0) u_cur = sched_grab(a.err);
    u_cur = __shfl_sync(0xffffffffu, u_cur, 0);
    if (lane == 0 && u_cur < units) u_nxt = sched_grab(a.err);
    u_nxt = u_cur < units ? __shfl_sync(0xffffffffu, u_nxt, 0) : units;
    Sched Sc, Sn;
    bool ok = issue_group(u_cur, 0, Sc);
    int ti = 0;
    for (int gi = 0; ok && u_cur < units; ++gi) {
      if (!issue_group(u_nxt, gi + 1, Sn)) {
        ok = false;
        break;
      }
      int u_after = units;  // read back (and so completed) at the end of the iteration on every path
      if (lane == 0 && u_nxt < units) u_after = sched_grab(a.err);
      const Sched S = Sc;
      if (S.active) {
        const int n_rec = S.n_ring + S.n_new;
        for (int i = 0; i < S.nh; ++i, ++ti) {
          const bool skp = (S.skip >> i) & 1u;  // decay-aware skip: no checkpoint tile for this head
          const bool hold = ti == a.withhold;  // test hook: this stage is never filled
          const uint32_t tbytes = (skp ? 0u : (uint32_t)lay.tile_bytes) + n_rec * xrow;
          const int s = ti % NS;
          if (!mbar_wait_or_abort(&empty[s], (uint32_t)(((ti / NS) & 1) ^ 1), abort_flag, ws)) {
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
          if (hold) continue;
          if (lane == 0 && !skp) bulk_g2s(st, a.hp + unit * a.P * kCols, lay.tile_bytes, &full[s], pol_stream);
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
      Sc = Sn;
      u_cur = u_nxt;
      u_nxt = __shfl_sync(0xffffffffu, u_after, 0);
    }
    if (!ok && lane == 0) {
      record_error(a.err, 0, RSSM_DEV_TIMEOUT);
      *abort_flag = 1;
    }
  } else if (warp == kPrepWarp) {
    // ================================================================== prep warp
    for (int gi = 0;; ++gi) {
      const int gs = gi % kGB, tsl = gi & 1;
      if (!mbar_wait_or_abort(&gfull[gs], (uint32_t)((gi / kGB) & 1), abort_flag, ws) ||
          !mbar_wait_or_abort(&tempty[tsl], (uint32_t)(((gi >> 1) & 1) ^ 1), abort_flag, ws)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      const unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      if (gh[G_END]) {  // no more units: let the consumers see the marker
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[tsl]);
        break;
      }
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
        if constexpr (kMma) {
          // g[j][r] = B_r . C_j on tensor cores (both exact in bf16): rows = outputs (8 of 16), columns =
          // 8 records per tile, 8 k-steps of 16 state columns
          const int gq = lane >> 2, tq = lane & 3;
          uint32_t ca[8][2];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const TI *cr = Cg + gq * kCols + 16 * c + 2 * tq;
            ca[c][0] = gq < t_out ? *reinterpret_cast<const uint32_t *>(cr) : 0u;
            ca[c][1] = gq < t_out ? *reinterpret_cast<const uint32_t *>(cr + 8) : 0u;
          }
          for (int r0 = 0; r0 < n_rec; r0 += 8) {
            const TI *br = Bg + (size_t)min(r0 + gq, n_rec - 1) * kCols + 2 * tq;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 8; ++c)
              mma_16816(d, ca[c][0], 0u, ca[c][1], 0u, *reinterpret_cast<const uint32_t *>(br + 16 * c),
                        *reinterpret_cast<const uint32_t *>(br + 16 * c + 8));
            const int r = r0 + 2 * tq;
            if (r < n_rec) T.g[gq * rmax + r] = d[0];
            if (r + 1 < n_rec) T.g[gq * rmax + r + 1] = d[1];
          }
        } else {
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
        // dt of the new tokens goes to each head's ring row
        for (int q = lane; q < n_new * nh; q += 32) {
          const int t = q / nh, i = q % nh;
          a.ring_dt[((size_t)b * a.H + h0 + i) * dts + slot0 + t] = gf[G_DT + t * kHG + i];
        }
        __syncwarp();
        // per-head weights of every record in every output (log-space suffix sums of dt):
        // coef[r] = dt_r exp(A s(r+1, e_j)) (B_r . C_j) for m <= r < e_j, plus D on the output's
        // own token r = e_j - 1, and 0 elsewhere; ao = exp(A s(m, e_j)) scales S' C_j
        if constexpr (kMma) {
          // per head, T[x] = sum of dt over records x .. n_rec - 1 (records below m left out), by a reverse
          // warp scan over lanes x and x + 32.  Record r weighs dt_r exp(A (T[r+1] - T[e_j])) (B_r . C_j) in
          // output j for m <= r < e_j, plus D on r = e_j - 1, and ao_j = exp(A (T[m] - T[e_j])).  Lane 4j + t
          // writes its fragment slot of every 16-record step (records 16q + 2t + {0, 1, 8, 9}) as bf16 hi
          // and lo words.
          const int jl = lane >> 2, tl = lane & 3;
          const int e_l = n_rec - t_out + jl + 1;
          const bool jv = jl < t_out;
          for (int i = 0; i < nh; ++i) {
            const float A = gf[G_A + i];
            const float dlo = (lane >= m && lane < n_rec) ? dt_of(i, lane) : 0.f;
            const float dhi = (lane + 32 >= m && lane + 32 < n_rec) ? dt_of(i, lane + 32) : 0.f;
            float tlo = dlo, thi = dhi;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
              const float vlo = __shfl_down_sync(0xffffffffu, tlo, off);
              const float vhi = __shfl_down_sync(0xffffffffu, thi, off);
              if (lane + off < 32) {
                tlo += vlo;
                thi += vhi;
              }
            }
            tlo += __shfl_sync(0xffffffffu, thi, 0);
            auto at = [&](float lo, float hi, int x) -> float {  // value of lane x of the 64-lane pair
              const float a0 = __shfl_sync(0xffffffffu, lo, x & 31), a1 = __shfl_sync(0xffffffffu, hi, x & 31);
              return x < 32 ? a0 : a1;
            };
            const float Te = at(tlo, thi, e_l), Tm = at(tlo, thi, m);
            if (jv && tl == 0) T.ao[i * NO + jl] = __expf(A * (Tm - Te));
            uint4 *cf = reinterpret_cast<uint4 *>(T.coef) + (size_t)i * lay.nq * 32;
            for (int q = 0; q < lay.nq; ++q) {
              float co[4];
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                const int r = 16 * q + 2 * tl + (z & 1) + 8 * (z >> 1);
                const float Tn = at(tlo, thi, r + 1), dr = at(dlo, dhi, r);
                float v = 0.f;
                if (jv && r >= m && r < e_l) v = dr * __expf(A * (Tn - Te)) * T.g[jl * rmax + r];
                if (jv && r == e_l - 1) v += gf[G_D + i];
                co[z] = v;
              }
              uint4 w;
              split_bf16x2(co[0], co[1], w.x, w.z);
              split_bf16x2(co[2], co[3], w.y, w.w);
              cf[q * 32 + lane] = w;
            }
          }
        } else {
          for (int pr = lane; pr < nh * t_out; pr += 32) {
            const int i = pr / t_out, j = pr % t_out;
            const float A = gf[G_A + i];
            const int e_j = n_rec - t_out + j + 1;
            float sfx = 0.f;
            float *co = T.coef + (i * NO + j) * rmax;
            for (int r = e_j; r < n_rec; ++r) co[r] = 0.f;
            for (int r = e_j - 1; r >= m; --r) {
              const float d = dt_of(i, r);
              co[r] = d * __expf(A * sfx) * T.g[j * rmax + r];
              sfx += d;
            }
            for (int r = 0; r < m; ++r) co[r] = 0.f;
            co[e_j - 1] += gf[G_D + i];
            T.ao[i * NO + j] = __expf(A * sfx);
          }
        }
        if (a.skip != nullptr && lane < nh) {
          // skip flag for the next call: A_h times the fp32 sum of dt, in record order, over the records
          // committed after this call (records m.. ; a verify's drafts are not committed)
          const int n_comm = a.op == OP_VERIFY ? n_ring : n_rec;
          float sdt = 0.f;
          for (int r = m; r < n_comm; ++r) sdt = __fadd_rn(sdt, dt_of(lane, r));
          a.skip[(size_t)b * a.H + h0 + lane] = __fmul_rn(gf[G_A + lane], sdt) < a.skip_ln_tau ? 1 : 0;
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
      if (TCF && lay.tb_bk > 0 && gh[G_ACTIVE] && gh[G_M] > 0) {
        // the folded B records (r < m) as the chunked fold's B operand: in each 16-column chunk, columns
        // {0,1,4,5,8,9,12,13} then {2,3,6,7,10,11,14,15} (bf16 pairs stay together), at a pitch of 272 bytes
        const int mf = gh[G_M];
        unsigned char *bk = tabs + (size_t)tsl * lay.tab_bytes + lay.tb_bk;
        for (int q = lane; q < mf * 8; q += 32) {
          const int r = q >> 3, c = q & 7;
          const uint4 *src = reinterpret_cast<const uint4 *>(gb + lay.gb_B + (size_t)r * kCols * 2 + c * 32);
          const uint4 w0 = src[0], w1 = src[1];
          uint4 *dst = reinterpret_cast<uint4 *>(bk + (size_t)r * kBkPitch + c * 32);
          dst[0] = make_uint4(w0.x, w0.z, w1.x, w1.z);
          dst[1] = make_uint4(w0.y, w0.w, w1.y, w1.w);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfull[tsl]);
    }
  } else {
    // ================================================================== consumer warps
    const int row0 = warp * 8;
    const uint64_t pol_ring = policy_evict_last();
    int ti = 0;
    int cft = 0;  // chunked fold tiles seen (every consumer warp sees every tile)
    for (int gi = 0;; ++gi) {
      const int gs = gi % kGB, tsl = gi & 1;
      if (!mbar_wait_or_abort(&tfull[tsl], (uint32_t)((gi >> 1) & 1), abort_flag, ws)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      const unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      if (gh[G_END]) break;
      const int b = gh[G_B], h0 = gh[G_H0], nh = gh[G_NH];
      if (gh[G_ACTIVE]) {
        const Tables T = tables(tsl);
        const float *t_coef = T.coef, *t_ao = T.ao, *t_wf = T.wf, *t_af = T.af;
        const int n_rec = gh[G_NREC], m = gh[G_M], t_out = gh[G_TOUT];
        const int n_ring = gh[G_NRING], n_new = gh[G_NNEW], slot0 = gh[G_SLOT0];
        const unsigned skm = (unsigned)gh[G_SKIP];
        const TI *Bg = reinterpret_cast<const TI *>(gb + lay.gb_B);
        const TI *Cg = reinterpret_cast<const TI *>(gb + lay.gb_C);
        // ---- stream the heads' tiles; each warp works and releases on its own
        float4 cv[kMma ? 1 : NO];
        // tensor-core path: C_j as the B operand of eight 16-column steps (column j = lane / 4;
        // lane 4g + t holds columns 16c + 4t .. 16c + 4t + 3 of step c, the k order the S' loads use)
        uint32_t ac[kMma ? 8 : 1][2];
        if constexpr (kMma) {
          const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint2 v = make_uint2(0u, 0u);
            if (g < t_out) v = *reinterpret_cast<const uint2 *>(Cg + g * kCols + 16 * c + 4 * t4);
            ac[c][0] = v.x;
            ac[c][1] = v.y;
          }
        } else {
#pragma unroll
          for (int j = 0; j < NO; ++j) cv[j] = (j < t_out) ? load4(Cg + j * kCols + 4 * lane) : make_float4(0, 0, 0, 0);
        }
        constexpr int V = 8 * NO;
        constexpr int KEEP = V >= 32 ? V / 32 : 1;
        constexpr int SPREAD = V >= 32 ? 1 : 32 / V;
        for (int i = 0; i < nh; ++i, ++ti) {
          const int s = ti % NS;
          if (!mbar_wait_or_abort(&full[s], (uint32_t)((ti / NS) & 1), abort_flag, ws)) {
            if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
            break;
          }
          const unsigned char *st = stages + (size_t)s * lay.stage_bytes;
          const float *tile = reinterpret_cast<const float *>(st);
          const TI *xr = reinterpret_cast<const TI *>(st + lay.xr);
          const int h = h0 + i;
          const size_t unit = (size_t)b * a.H + h;
          // a fold tile of the chunked form is taken by one group of four warps (alternating); the other group
          // only waits for it to land (so that its release cannot count for the stage's previous use)
          const bool gtile = TCF && lay.tb_bk > 0 && m > 0;
          const int grp = cft & 1;
          cft += gtile ? 1 : 0;
          const bool mine = !gtile || (warp >> 2) == grp;
          // the new tokens' x rows, landed in the stage behind the buffered ones, go to the head's
          // ring row with one bulk store (warps take turns); the stage is released after it has
          // been read
          const bool appender = (gtile ? 4 * grp + (ti & 3) : (ti & (kConsumerWarps - 1))) == warp && n_new > 0;
          if (appender && lane == 0) {
            const uint32_t xrow = (uint32_t)a.P * esz;
            bulk_s2g(reinterpret_cast<unsigned char *>(a.ring_x) + (unit * 2 * a.L + slot0) * xrow,
                     st + lay.xr + (size_t)n_ring * xrow, (uint32_t)n_new * xrow, pol_ring);
            bulk_commit();
          }
          if (!mine) {
          } else if (gtile) {
            // ---- chunked fold: S' = af S + X' B with X'[row][r] = wf_r x_r[row] (r < m <= 16) on the tensor
            // cores.  Warp (w & 3) of the group owns rows 16(w & 3) .. +15; lane 4g+t holds rows ra = .. + g and
            // rb = ra + 8 and, in each 16-column chunk c, the columns 16c + 4t .. +3, which the reordered B
            // records match as fragments.  X' is cut into three bf16 pieces whose sum is exact; B is exact.
            const int gq = lane >> 2, qtr = lane & 3, odd = gq & 1;
            const int ra = 16 * (warp & 3) + gq, rb = ra + 8;
            const bool va = ra < a.P, vb = rb < a.P;
            const bool skp = (skm >> i) & 1u;  // a skipped head folds from zero
            const bool la = va && !skp, lb = vb && !skp;
            float *tw = const_cast<float *>(tile);
            auto srow = [&](int r, int c) { return reinterpret_cast<float4 *>(tw + (size_t)r * kCols + 16 * c + 4 * qtr); };
            float xa4[4], xb4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int r = 2 * qtr + (k & 1) + 8 * (k >> 1);
              float u = 0.f, v = 0.f;
              if (r < m) {
                const float wr = t_wf[i * rmax + r];
                if (va) u = wr * to_f32(xr[r * a.P + ra]);
                if (vb) v = wr * to_f32(xr[r * a.P + rb]);
              }
              xa4[k] = u;
              xb4[k] = v;
            }
            uint32_t wp[3][4];
            split3_bf16x2(xa4[0], xa4[1], wp[0][0], wp[1][0], wp[2][0]);
            split3_bf16x2(xb4[0], xb4[1], wp[0][1], wp[1][1], wp[2][1]);
            split3_bf16x2(xa4[2], xa4[3], wp[0][2], wp[1][2], wp[2][2]);
            split3_bf16x2(xb4[2], xb4[3], wp[0][3], wp[1][3], wp[2][3]);
            const float af = t_af[i];
            const unsigned char *kt = tabs + (size_t)tsl * lay.tab_bytes + lay.tb_bk +
                                      (size_t)min((lane & 7) + 8 * ((lane >> 3) & 1), m - 1) * kBkPitch + (lane >> 4) * 16;
            float *dst = a.hp + unit * a.P * kCols;
#pragma unroll
            for (int cp = 0; cp < 8; cp += 2) {
              // rows of odd g take the chunk pair in the other order: no bank conflicts
              const int c0 = cp + odd, c1 = cp + 1 - odd;
              float4 xa[2], xb[2];
              {
                const float4 pa = la ? *srow(ra, c0) : f4zero(), pb = lb ? *srow(rb, c0) : f4zero();
                const float4 qa = la ? *srow(ra, c1) : f4zero(), qb = lb ? *srow(rb, c1) : f4zero();
                xa[0] = odd ? qa : pa; xa[1] = odd ? pa : qa;
                xb[0] = odd ? qb : pb; xb[1] = odd ? pb : qb;
              }
#pragma unroll
              for (int o2 = 0; o2 < 2; ++o2) {
                uint32_t q0, q1, q2, q3;  // n-tile (chunk, 0): q0 (records 0-7), q1 (8-15); (chunk, 1): q2, q3
                ldmatrix_x4_trans(kt + (cp + o2) * 32, q0, q1, q2, q3);
#pragma unroll
                for (int o = 0; o < 2; ++o) {
                  float d[4];
                  if (o == 0) { d[0] = xa[o2].x * af; d[1] = xa[o2].y * af; d[2] = xb[o2].x * af; d[3] = xb[o2].y * af; }
                  else        { d[0] = xa[o2].z * af; d[1] = xa[o2].w * af; d[2] = xb[o2].z * af; d[3] = xb[o2].w * af; }
#pragma unroll
                  for (int pz = 2; pz >= 0; --pz) mma_16816(d, wp[pz][0], wp[pz][1], wp[pz][2], wp[pz][3], o ? q2 : q0, o ? q3 : q1);
                  if (o == 0) { xa[o2].x = d[0]; xa[o2].y = d[1]; xb[o2].x = d[2]; xb[o2].y = d[3]; }
                  else        { xa[o2].z = d[0]; xa[o2].w = d[1]; xb[o2].z = d[2]; xb[o2].w = d[3]; }
                }
              }
              if (va) {
                *srow(ra, c0) = odd ? xa[1] : xa[0];
                *srow(ra, c1) = odd ? xa[0] : xa[1];
                __stcs(reinterpret_cast<float4 *>(dst + (size_t)ra * kCols + 16 * cp + 4 * qtr), xa[0]);
                __stcs(reinterpret_cast<float4 *>(dst + (size_t)ra * kCols + 16 * (cp + 1) + 4 * qtr), xa[1]);
              }
              if (vb) {
                *srow(rb, c0) = odd ? xb[1] : xb[0];
                *srow(rb, c1) = odd ? xb[0] : xb[1];
                __stcs(reinterpret_cast<float4 *>(dst + (size_t)rb * kCols + 16 * cp + 4 * qtr), xb[0]);
                __stcs(reinterpret_cast<float4 *>(dst + (size_t)rb * kCols + 16 * (cp + 1) + 4 * qtr), xb[1]);
              }
            }
            if constexpr (kMma) {
              // 8 outputs on the tensor cores, as on the streaming path but for the group's 16 rows: S' (read back,
              // each lane its own values) in bf16 hi and lo pieces times [C_1 .. C_8], then the buffered term
              // [x_r] times the coefficient fragments of the prep warp
              float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float4 sa = va ? *srow(ra, c) : f4zero(), sb = vb ? *srow(rb, c) : f4zero();
                uint32_t h0, l0, h1, l1, h2, l2, h3, l3;
                split_bf16x2(sa.x, sa.y, h0, l0);
                split_bf16x2(sb.x, sb.y, h1, l1);
                split_bf16x2(sa.z, sa.w, h2, l2);
                split_bf16x2(sb.z, sb.w, h3, l3);
                mma_16816(d1, l0, l1, l2, l3, ac[c][0], ac[c][1]);
                mma_16816(d0, h0, h1, h2, h3, ac[c][0], ac[c][1]);
              }
              float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
              const uint4 *cf = reinterpret_cast<const uint4 *>(t_coef) + (size_t)i * lay.nq * 32;
              const unsigned short *xs = reinterpret_cast<const unsigned short *>(xr);
              for (int q = 0; q * 16 < n_rec; ++q) {
                const uint4 w = cf[q * 32 + lane];
                const int r0 = 16 * q + 2 * qtr;
                auto xw = [&](int r, int row, bool v) -> uint32_t { return (v && r < n_rec) ? xs[r * a.P + row] : 0u; };
                const uint32_t xa0 = xw(r0, ra, va) | (xw(r0 + 1, ra, va) << 16);
                const uint32_t xb0 = xw(r0, rb, vb) | (xw(r0 + 1, rb, vb) << 16);
                const uint32_t xa8 = xw(r0 + 8, ra, va) | (xw(r0 + 9, ra, va) << 16);
                const uint32_t xb8 = xw(r0 + 8, rb, vb) | (xw(r0 + 9, rb, vb) << 16);
                mma_16816(e0, xa0, xb0, xa8, xb8, w.x, w.y);
                mma_16816(e1, xa0, xb0, xa8, xb8, w.z, w.w);
              }
              const int j0 = 2 * qtr;
              const size_t jstride = (size_t)a.H * a.P;
              float *yo = a.y + (((size_t)b * a.T + j0) * a.H + h) * a.P;
              if (j0 < t_out) {
                const float ao = t_ao[i * NO + j0];
                if (va) yo[ra] = ao * (d0[0] + d1[0]) + (e0[0] + e1[0]);
                if (vb) yo[rb] = ao * (d0[2] + d1[2]) + (e0[2] + e1[2]);
              }
              if (j0 + 1 < t_out) {
                const float ao = t_ao[i * NO + j0 + 1];
                if (va) yo[jstride + ra] = ao * (d0[1] + d1[1]) + (e0[1] + e1[1]);
                if (vb) yo[jstride + rb] = ao * (d0[3] + d1[3]) + (e0[3] + e1[3]);
              }
            } else {
              // outputs from S' (each lane reads back what it wrote): ao_j (S' . C_j) + sum_r coef_jr x_r[row]
              for (int j = 0; j < t_out; ++j) {
                float ya = 0.f, yb = 0.f;
  #pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const int cc = c ^ odd;  // odd rows in the other chunk order, as written
                  const float4 cj = load4(Cg + j * kCols + 16 * cc + 4 * qtr);
                  if (va) {
                    const float4 sa = *srow(ra, cc);
                    ya = fmaf(sa.x, cj.x, fmaf(sa.y, cj.y, fmaf(sa.z, cj.z, fmaf(sa.w, cj.w, ya))));
                  }
                  if (vb) {
                    const float4 sb = *srow(rb, cc);
                    yb = fmaf(sb.x, cj.x, fmaf(sb.y, cj.y, fmaf(sb.z, cj.z, fmaf(sb.w, cj.w, yb))));
                  }
                }
                const float ao = t_ao[i * NO + j];
                ya *= ao;
                yb *= ao;
                for (int r = qtr; r < n_rec; r += 4) {
                  const float co = t_coef[(i * NO + j) * rmax + r];
                  if (va) ya = fmaf(co, to_f32(xr[r * a.P + ra]), ya);
                  if (vb) yb = fmaf(co, to_f32(xr[r * a.P + rb]), yb);
                }
                ya += __shfl_xor_sync(0xffffffffu, ya, 1);
                yb += __shfl_xor_sync(0xffffffffu, yb, 1);
                ya += __shfl_xor_sync(0xffffffffu, ya, 2);
                yb += __shfl_xor_sync(0xffffffffu, yb, 2);
                float *yj = a.y + (((size_t)b * a.T + j) * a.H + h) * a.P;
                if (qtr == 0 && va) yj[ra] = ya;
                if (qtr == 0 && vb) yj[rb] = yb;
              }
            }
          } else if (row0 < a.P) {
            // a head flagged for decay-aware skipping has no tile in the stage: its checkpoint term is zero
            const bool skp = (skm >> i) & 1u;
            float4 sv[8];
            if (!kMma || m > 0) {
#pragma unroll
            for (int rr = 0; rr < 8; ++rr)
              sv[rr] = skp ? make_float4(0.f, 0.f, 0.f, 0.f)
                           : *reinterpret_cast<const float4 *>(tile + (row0 + rr) * kCols + 4 * lane);
            }
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
              if constexpr (kMma) {  // the folded rows replace this warp's rows of the stage
                float *tw = const_cast<float *>(tile);
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) *reinterpret_cast<float4 *>(tw + (row0 + rr) * kCols + 4 * lane) = sv[rr];
                fence_async_smem();  // ordered before the stage's next bulk fill
                __syncwarp();
              }
            }
            if constexpr (kMma) {
              if (t_out > 0) {
                // D[16 x 8] = [S'_hi; S'_lo] (the warp's 8 state rows, split into bf16 hi and lo
                // halves as rows 0-7 and 8-15) times [C_1 .. C_T] over 8 k-steps of 16 state
                // columns, in two independent accumulators; lane 4g + t then holds rows
                // p = row0 + g, outputs j = 2t, 2t + 1 of both halves.  The buffered term
                // sum_r x_r[p] coef_{j,r} follows as [x_r (exact bf16); 0] times the coefficient
                // split into hi + lo, over 16-record steps.
                const int g = lane >> 2, t4 = lane & 3;
                float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
                const float *srow = tile + (row0 + g) * kCols + 4 * t4;
                if (!skp || m > 0) {  // a skipped head's folded rows were written back into the stage
#pragma unroll
                  for (int c = 0; c < 8; ++c) {
                    const float4 v = *reinterpret_cast<const float4 *>(srow + 16 * c);
                    uint32_t h0, l0, h1, l1;
                    split_bf16x2(v.x, v.y, h0, l0);
                    split_bf16x2(v.z, v.w, h1, l1);
                    mma_16816((c & 1) ? d1 : d0, h0, l0, h1, l1, ac[c][0], ac[c][1]);
                  }
                }
                float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
                const uint4 *cf = reinterpret_cast<const uint4 *>(t_coef) + (size_t)i * lay.nq * 32;
                const unsigned short *xs = reinterpret_cast<const unsigned short *>(xr) + row0 + g;
                for (int q = 0; q * 16 < n_rec; ++q) {
                  const uint4 w = cf[q * 32 + lane];
                  const int r0 = 16 * q + 2 * t4;
                  const uint32_t x0 = r0 < n_rec ? xs[r0 * a.P] : 0u, x1 = r0 + 1 < n_rec ? xs[(r0 + 1) * a.P] : 0u;
                  const uint32_t x8 = r0 + 8 < n_rec ? xs[(r0 + 8) * a.P] : 0u;
                  const uint32_t x9 = r0 + 9 < n_rec ? xs[(r0 + 9) * a.P] : 0u;
                  const uint32_t xa = x0 | (x1 << 16), xb = x8 | (x9 << 16);
                  mma_16816(e0, xa, 0u, xb, 0u, w.x, w.y);
                  mma_16816(e1, xa, 0u, xb, 0u, w.z, w.w);
                }
                const int j0 = 2 * t4;
                float *yo = a.y + (((size_t)b * a.T + j0) * a.H + h) * a.P + row0 + g;
                const size_t jstride = (size_t)a.H * a.P;
                if (j0 < t_out)
                  yo[0] = t_ao[i * NO + j0] * ((d0[0] + d1[0]) + (d0[2] + d1[2])) + (e0[0] + e1[0]);
                if (j0 + 1 < t_out)
                  yo[jstride] = t_ao[i * NO + j0 + 1] * ((d0[1] + d1[1]) + (d0[3] + d1[3])) + (e0[1] + e1[1]);
              }
            } else {
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
          }
          if (appender && lane == 0) bulk_wait_read();
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
    if (lane == 0) bulk_wait_all();
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // do not leave bulk copies in flight into the shared memory of an exiting block
    for (int s = 0; s < 8; ++s)
      if (armed[s] >= 0) mbar_wait(&full[s], (uint32_t)(armed[s] & 1), ws);
    for (int s = 0; s < kGB; ++s)
      if (armed[8 + s] >= 0) mbar_wait(&gfull[s], (uint32_t)(armed[8 + s] & 1), ws);
  }
  if (threadIdx.x == 0) sched_finish(a.err);
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
  if (no == NOV) kern = m2_replay_kernel<TI, NOV, false>;
  if (esz == 2) {
    RSSM_PICK(__nv_bfloat16, 1) RSSM_PICK(__nv_bfloat16, 2) RSSM_PICK(__nv_bfloat16, 4) RSSM_PICK(__nv_bfloat16, 8)
    if (no == 1 && !a.fold_free) kern = m2_replay_kernel<__nv_bfloat16, 1, true>;
    if (no == 8) kern = m2_replay_kernel<__nv_bfloat16, 8, true>;
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
