// gdn.cu -- ReplaySSM decode kernels for Gated DeltaNet layers (sm_100a).
//
// Per (sequence b, head h) the state S in R^{d_v x 128} follows the gated delta rule
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   y_t = q_scale S_t q_t
// and is held as a checkpoint plus the inputs (k, v, alpha, beta) of the tokens since it
// ("SSM decoding stops writing state every step", Synopsis and Interpretation, second
// paragraph).  With the call's records r = 0..n_rec-1 (buffered, then new), the first m
// are folded into the state and output j replays records m..e_j-1.  The replay walks q
// back through the buffered factors, newest first:
//     u <- q_j;  for r = e_j-1 .. m:  c_r = k_r . u;  u <- alpha_r (u - beta_r c_r k_r)
//     y_j = q_scale (S' u + sum_r beta_r c_r v_r)
// so the checkpoint enters through one matrix-vector product per output.  The fold is
// row-local: each row s of S takes, record by record,
//     s <- alpha_r s + beta_r (v_r[row] - alpha_r (s . k_r)) k_r.
//
// Precision modes ("Hybrid-model decoding has a new bottleneck", Interpretation, fourth
// paragraph, Perspective, second paragraph; FP8: "SSM decoding stops writing state every
// step", Interpretation, third paragraph): the checkpoint is fp32, fp16 written with
// stochastic rounding, or E4M3 times a per-tile fp32 scale written the same way; the copy
// read by non-fold outputs is the checkpoint itself, a separate NVFP4 copy re-quantised
// from the fp32 fold result, or (contrast) an NVFP4 copy that is also the state the
// recurrence continues from.  Outputs of a call that folds come from the fp32 fold result.
//
// Decay-aware read skipping ("SSM decoding stops writing state every step", Perspective,
// first paragraph): with a threshold tau > 0, a head whose alpha product over the
// committed records of its window is below tau (fp32, record order; decided by the prep
// warps at the end of a call) skips the next call's checkpoint read: no tile copy, a zero
// term, and a fold from zero.
//
// Block roles (one block per SM, persistent; units drawn from a per-launch counter):
//  * producer warp: TMA bulk copies (cp.async.bulk) of each unit's k records, q and
//    alpha/beta rows into one of three group buffers, one unit ahead of the unit whose
//    tiles it is issuing, and of each 64-row tile of a head's state (in its stored
//    format) plus the head's v records into a ring of stages (the head's first tile
//    stage also feeds the bulk store that appends its new v rows);
//  * two prep warps: 8-lane subgroups walk q back for every (head, draft) pair of the
//    unit, writing u_0 and the coefficients beta_r c_r into double-buffered tables;
//    they also append k, alpha, beta of the new tokens and write the bookkeeping word;
//  * eight consumer warps take every tile, warp w rows 8w..8w+7.  Non-fold tiles: lane l
//    owns columns 4l..4l+3, the row dot products with u_0 and the buffered term finish in
//    one warp transpose reduction.  Fold tiles: four lanes own one row (32 columns each,
//    in registers) and run the sequential row update with two shuffles per record; then
//    the new state is written in the checkpoint format and, in E4M3 and NVFP4 modes,
//    quantised (tile maximum over the eight warps through an mbarrier rendezvous with
//    bounded waits).
// Work unit: (sequence, chunk of HG heads), HG = 4, 4, 2, 1 for 1, 2, 4, 8 outputs.
#include "common.cuh"
#include "kernels.h"
#include "lowprec.cuh"

namespace rssm {

namespace {

constexpr int kGHdrBytes = 1024;
enum {
  Q_ACTIVE = 0, Q_NREC, Q_M, Q_NRING, Q_NNEW, Q_TOUT, Q_SLOT0, Q_MC, Q_ME, Q_MP, Q_B, Q_H0, Q_NH, Q_BASE,
  Q_WMETA, Q_SKIP, Q_END,  // Q_SKIP: bit i set = head h0 + i skips its checkpoint read in this call
  Q_F = 32,                // floats: alpha of new tokens [8][8] (token, head)
  Q_FB = Q_F + 64          // beta of new tokens [8][8]
};
constexpr int kGdnThreads = kConsumers + 96;  // + producer + two prep warps
constexpr int kGProducer = kConsumerWarps, kGPrep0 = kConsumerWarps + 1;
constexpr int kTileMaxBytes = kFp4Rows * kCols * 4;  // a 64-row fp32 tile

__host__ __device__ inline int g_heads_per_unit(int no) { return no == 1 ? 4 : no == 2 ? 4 : no == 4 ? 2 : 1; }

// Chunked fold.  Folding m records into a row s of the state is, with a_r = prod_{j<=r} alpha_j,
// b_r = prod_{r<j<m} alpha_j, z_r = s . k_r and u the per-record coefficients of the sequential rule,
//     u = T rt,  rt_r = beta_r (v_r[row] - a_r z_r),  T = (I + L)^-1,
//     L_ri = beta_r (prod_{i<j<=r} alpha_j) (k_i . k_r)  (i < r),
//     s' = a_{m-1} s + sum_r b_r u_r k_r,
// the rank-m form of the delta rule's product of elementary factors.  For an fp32 checkpoint with bf16
// inputs and m <= kChMax the consumers run it on the tensor cores per 16-row block: Z = S K^T, U = RT T^T and
// S' = a_{m-1} S + W K with W = b U, each fp32 operand cut into three bf16 pieces whose sum is exact.  Per
// head the prep warps leave T (16 x 16, zero past m), a_r and b_r in the tables, and reorder the folded K rows
// in the group buffer (pitch 272 bytes) so that both K operands load with ldmatrix, free of bank conflicts.
constexpr int kChMax = 16;
constexpr int kChT = kChMax * kChMax;               // T[r][i], row-major
constexpr int kChStride = kChT + 2 * kChMax + 4;    // per head: T, a_r, b_r (+4: heads in different banks)
// the checkpoint formats and window for which folds take the chunked form: an fp32 checkpoint, read as it is
// or through the NVFP4 copy (re-quantised from the chunked result), with bf16 inputs
__host__ __device__ inline bool g_chunked(int hp_mode, int read_mode, int esz, int L) {
  return hp_mode == RSSM_HP_F32 && (read_mode == RSSM_READ_SAME || read_mode == RSSM_READ_NVFP4) && esz == 2 &&
         L <= kChMax;
}

struct GLayout {
  int no, rmax, hg, nrb, dts, kpe;        // kpe: element pitch of the K rows in the group buffer
  int gb_k, gb_q, gb_a, gb_b, gb_bytes;   // group buffer
  int tb_u0, tb_coef, tb_ab, tb_amax, tb_ch, tab_bytes; // tables (per buffer)
  int st_g, st_v, stage_bytes;            // tile stage: [tile 32 KiB][g chunk 16 B][v records]
};

__host__ __device__ inline GLayout g_layout(int R, int L, int tmax, int esz, bool chunk) {
  GLayout l;
  l.no = tmax <= 1 ? 1 : tmax <= 2 ? 2 : tmax <= 4 ? 4 : 8;
  l.rmax = L + (tmax > 1 ? tmax : 1);
  l.hg = g_heads_per_unit(l.no);
  l.nrb = (R + kFp4Rows - 1) / kFp4Rows;
  l.dts = dt_stride(L);
  l.kpe = kCols + (chunk ? 16 / esz : 0);
  l.gb_k = kGHdrBytes;
  l.gb_q = (int)align_up((size_t)l.gb_k + (size_t)l.hg * l.rmax * l.kpe * esz, 16);
  l.gb_a = (int)align_up((size_t)l.gb_q + (size_t)l.hg * l.no * kCols * esz, 16);
  l.gb_b = l.gb_a + l.hg * l.dts * 4;
  l.gb_bytes = (int)align_up((size_t)l.gb_b + (size_t)l.hg * l.dts * 4, 128);
  l.tb_u0 = 0;
  l.tb_coef = l.hg * l.no * kCols * 4;
  l.tb_ab = (int)align_up((size_t)l.tb_coef + (size_t)l.hg * l.no * l.rmax * 4, 16);  // {a, b, 1/a, 0}[hg][rmax]
  l.tb_amax = l.tb_ab + l.hg * l.rmax * 16;
  l.tb_ch = l.tb_amax + 2 * 8 * 4;                                    // amax[slot][warp]
  l.tab_bytes = (int)align_up((size_t)l.tb_ch + (chunk ? (size_t)l.hg * kChStride * 4 : 0), 128);
  l.st_g = kTileMaxBytes;
  l.st_v = l.st_g + 16;
  l.stage_bytes = (int)align_up((size_t)l.st_v + (size_t)l.rmax * R * esz, 128);
  return l;
}

constexpr int kBarBytesG = 512;  // mbarriers (31 x 8 B) + armed phases + abort flag
constexpr int kGBG = 3;  // group buffers: the producer loads a unit's group data one unit ahead

// tile source formats
enum { SRC_F32 = 0, SRC_F16 = 1, SRC_FP4 = 2, SRC_F8 = 3, SRC_FP4D = 4 };
// two-axis copy: where a tile's column-group scales land in a stage (after the row-block scales)
constexpr int kColScaleOff = kTileMaxBytes / 2 + 1024;
// fold scratch of the two-axis copy: column maxima of a tile in three rotating slots, then the tile's
// column-group steps (read by every consumer warp after a rendezvous)
constexpr int kCmSlotWords = (kFp4Rows / 16) * kCols;
constexpr int kCmBytes = 3 * kCmSlotWords * 4 + kCmSlotWords * 4;

// d[16x8] += a[16x8] b[8x8], tf32 in (fp32 registers whose low 13 bits are zero), fp32 accumulate.
// Lane 4g+t holds a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]}, b = {B[t][g], B[t+4][g]},
// d = {D[g][2t..2t+1], D[g+8][2t..2t+1]}.
__device__ __forceinline__ void mma_1688_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <typename TI>
__device__ __forceinline__ void load_k16(const TI *p, float (&o)[16]) {  // 16 consecutive elements
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 v = load4(p + 4 * q);
    o[4 * q] = v.x; o[4 * q + 1] = v.y; o[4 * q + 2] = v.z; o[4 * q + 3] = v.w;
  }
}

// LP: the context stores a low-precision checkpoint or keeps an NVFP4 read copy.  LP = false
// compiles the fp32-checkpoint path alone, with every format branch folded away.  CF: the instance with the
// chunked fold (fp32 checkpoint, bf16 inputs, read as it is or through the NVFP4 copy); steps the host knows to be
// fold-free take the instance without it, whose streaming path then compiles as it did before the chunked fold.
// Both fold correctly.
template <typename TI, int NO, bool LP, bool CF>
__global__ void __launch_bounds__(kGdnThreads, 1) gdn_replay_kernel(GArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int esz = sizeof(TI);
  constexpr bool kChunk = CF && sizeof(TI) == 2;
  const bool chunk = kChunk && g_chunked(a.hp_mode, a.read_mode, esz, a.L);  // every fold takes it (m <= L)
  const GLayout lay = g_layout(a.DV, a.L, a.tmax, esz, chunk);
  const int NS = a.nstage, R = a.DV, L = a.L, HG = lay.hg, nrb = lay.nrb, dts = lay.dts;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + 8;
  uint64_t *gfull = empty + 8;       // [kGBG] group data landed
  uint64_t *gempty = gfull + kGBG;   // [kGBG] consumers done with a unit's group data
  uint64_t *tfull = gempty + kGBG;   // [2] tables ready
  uint64_t *tempty = tfull + 2;      // [2] consumers done with the tables
  uint64_t *psync = tempty + 2;      // rendezvous of the two prep warps (count 2)
  uint64_t *fsync = psync + 1;       // rendezvous of the eight consumer warps (NVFP4 tile maximum)
  uint64_t *csync = fsync + 1;       // [2] rendezvous of a group of four (chunked fold, NVFP4 tile maximum)
  volatile int *armed = reinterpret_cast<volatile int *>(csync + 2);  // [8 + kGBG]
  volatile int *abort_flag = armed + 8 + kGBG;
  unsigned char *tabs = smem + kBarBytesG;
  unsigned char *gbuf = tabs + 2 * lay.tab_bytes;
  unsigned char *stages = gbuf + kGBG * lay.gb_bytes;
  unsigned int *cmx = reinterpret_cast<unsigned int *>(stages + (size_t)NS * lay.stage_bytes);  // two-axis copy only
  float *kvals = reinterpret_cast<float *>(cmx + 3 * kCmSlotWords);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitSpec ws{a.wait_cycles, a.suspend_ns};
  const int chunks = (a.H + HG - 1) / HG;
  const int units = a.Bt * chunks;
  const bool fp4_read = LP && a.read_mode != RSSM_READ_SAME;
  const bool shared_fp4 = LP && a.read_mode == RSSM_READ_SHARED_NVFP4;
  const bool fp4d = LP && a.read_mode == RSSM_READ_NVFP4D;
  const int read_fmt = fp4d ? SRC_FP4D : SRC_FP4;  // format of the read copy
  const bool hp16 = LP && a.hp_mode == RSSM_HP_F16_SR;
  const bool hp8 = LP && a.hp_mode == RSSM_HP_F8_SR;
  const int hp_fmt = hp16 ? SRC_F16 : hp8 ? SRC_F8 : SRC_F32;  // format of the stored checkpoint

  if (threadIdx.x == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int s = 0; s < kGBG; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], kConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kConsumerWarps);
    }
    mbar_init(psync, 2);
    mbar_init(fsync, kConsumerWarps);
    mbar_init(&csync[0], 4);
    mbar_init(&csync[1], 4);
    for (int s = 0; s < 8 + kGBG; ++s) armed[s] = -1;
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (fp4d)
    for (int q = threadIdx.x; q < 3 * kCmSlotWords; q += blockDim.x) cmx[q] = 0u;
  __syncthreads();

  if (warp == kGProducer) {
    // ================================================================== producer warp
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    const uint32_t krow = (uint32_t)kCols * esz, vrow = (uint32_t)R * esz;
    struct Sched {
      int b, h0, nh, active, n_ring, n_new, m, t_out, slot0, base_e;
      unsigned skip;
    };
    // schedule of unit u from the sequence's bookkeeping word; u >= units writes the end marker
    auto schedule = [&](int u, Sched &S, int *hdr) {
      if (u >= units) {
        S = Sched{};
        if (lane == 0) { hdr[Q_ACTIVE] = 0; hdr[Q_END] = 1; }
        return;
      }
      const int b = u / chunks, ch = u % chunks;
      S.b = b; S.h0 = ch * HG; S.nh = min(HG, a.H - S.h0);
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
        if (c == L) { n_ring = L; m = L; slot0 = base_n; c1 = 1; me = e + 1; }
        else { n_ring = c; m = 0; slot0 = base_e + c; c1 = c + 1; }
        if (c1 == L) { m = n_ring + 1; mc = 0; me = me + 1; }
        else mc = c1;
      } else if (a.op == OP_VERIFY) {
        n_new = a.T;
        t_out = a.T;
        mp = a.T;
        if (c + a.T > L) { n_ring = c; m = c; slot0 = base_n; mc = 0; me = e + 1; }
        else { n_ring = c; m = 0; slot0 = base_e + c; }
      } else {
        if (!msk || c == 0) active = 0;
        else { n_ring = c; m = c; mc = 0; me = e + 1; }
      }
      S.active = active; S.n_ring = n_ring; S.n_new = n_new; S.m = m; S.t_out = t_out; S.slot0 = slot0;
      S.base_e = base_e;
      S.skip = active ? skm : 0u;
      if (lane == 0) {
        hdr[Q_ACTIVE] = active; hdr[Q_NREC] = n_ring + n_new; hdr[Q_M] = m; hdr[Q_NRING] = n_ring;
        hdr[Q_NNEW] = n_new; hdr[Q_TOUT] = t_out; hdr[Q_SLOT0] = slot0; hdr[Q_MC] = mc; hdr[Q_ME] = me;
        hdr[Q_MP] = mp; hdr[Q_B] = b; hdr[Q_H0] = S.h0; hdr[Q_NH] = S.nh; hdr[Q_BASE] = base_e;
        hdr[Q_WMETA] = (S.h0 == 0); hdr[Q_SKIP] = (int)S.skip; hdr[Q_END] = 0;
      }
    };
    // group data of unit u: k records and q of every head, alpha / beta ring rows
    auto issue_group = [&](int u, int gi, Sched &S) -> bool {
      const int gs = gi % kGBG;
      if (!mbar_wait_or_abort(&gempty[gs], (uint32_t)(((gi / kGBG) & 1) ^ 1), abort_flag, ws)) return false;
      unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      schedule(u, S, reinterpret_cast<int *>(gb));
      __syncwarp();
      const int n_rec = S.n_ring + S.n_new, nh = S.nh;
      const uint32_t gbytes = S.active ? (uint32_t)(nh * (n_rec * krow + S.t_out * krow) + 2 * nh * dts * 4) : 0u;
      if (lane == 0) {
        armed[8 + gs] = gi / kGBG;
        mbar_arrive_expect_tx(&gfull[gs], gbytes);
      }
      __syncwarp();
      if (S.active) {
        // a unit that folds in the chunked form takes its K rows at the padded pitch (the ring part row by row)
        const bool krows = lay.kpe != kCols && S.m > 0;
        const uint32_t kp = krows ? (uint32_t)lay.kpe * esz : krow;
        const int nrc = krows ? S.n_ring : 1;  // copies of the ring part of a head's K rows
        const int per_head = nrc + S.n_new + S.t_out;
        const int ncopy = nh * per_head + 2;
        for (int q = lane; q < ncopy; q += 32) {
          if (q == ncopy - 2) {
            bulk_g2s(gb + lay.gb_a, a.ring_a + ((size_t)S.b * a.H + S.h0) * dts, nh * dts * 4, &gfull[gs], pol_keep);
          } else if (q == ncopy - 1) {
            bulk_g2s(gb + lay.gb_b, a.ring_b + ((size_t)S.b * a.H + S.h0) * dts, nh * dts * 4, &gfull[gs], pol_keep);
          } else {
            const int i = q / per_head, w = q % per_head;
            const size_t unit = (size_t)S.b * a.H + S.h0 + i;
            unsigned char *kd = gb + lay.gb_k + (size_t)i * lay.rmax * kp;
            if (w < nrc) {
              if (krows)
                bulk_g2s(kd + w * kp, reinterpret_cast<const unsigned char *>(a.ring_k) + (unit * 2 * L + S.base_e + w) * krow,
                         krow, &gfull[gs], pol_keep);
              else if (S.n_ring)
                bulk_g2s(kd, reinterpret_cast<const unsigned char *>(a.ring_k) + (unit * 2 * L + S.base_e) * krow,
                         S.n_ring * krow, &gfull[gs], pol_keep);
            } else if (w < nrc + S.n_new) {
              const int t = w - nrc;
              bulk_g2s(kd + (S.n_ring + t) * kp,
                       reinterpret_cast<const unsigned char *>(a.k) + (((size_t)S.b * a.T + t) * a.H + S.h0 + i) * krow,
                       krow, &gfull[gs], pol_keep);
            } else {
              const int t = w - nrc - S.n_new;
              bulk_g2s(gb + lay.gb_q + ((size_t)i * lay.no + t) * krow,
                       reinterpret_cast<const unsigned char *>(a.q) + (((size_t)S.b * a.T + t) * a.H + S.h0 + i) * krow,
                       krow, &gfull[gs], pol_keep);
            }
          }
        }
      }
      return true;
    };
    // units come from the launch's counter: the group data of the next unit is issued once the current
    // unit's first two tiles are on their way (its bookkeeping load then does not hold them up), and the
    // unit after that is requested (atomic in flight) meanwhile
    int u_cur = 0, u_nxt = 0;
    if (lane == 0) u_cur = sched_grab(a.err);
    u_cur = __shfl_sync(0xffffffffu, u_cur, 0);
    if (lane == 0 && u_cur < units) u_nxt = sched_grab(a.err);
    u_nxt = u_cur < units ? __shfl_sync(0xffffffffu, u_nxt, 0) : units;
    Sched Sc, Sn;
    bool ok = issue_group(u_cur, 0, Sc);
    int ti = 0;
    for (int gi = 0; ok && u_cur < units; ++gi) {
      int u_after = units;  // read back (and so completed) at the end of the iteration
      bool nxt_issued = false;
      auto issue_next = [&]() -> bool {
        nxt_issued = true;
        if (!issue_group(u_nxt, gi + 1, Sn)) return false;
        if (lane == 0 && u_nxt < units) u_after = sched_grab(a.err);
        return true;
      };
      const Sched S = Sc;
      if (S.active) {
        const int n_rec = S.n_ring + S.n_new;
        const bool fold = S.m > 0;
        const int srcfmt = fold ? (shared_fp4 ? SRC_FP4 : hp_fmt)
                                : (fp4_read ? read_fmt : hp_fmt);
        const bool fp4src = srcfmt == SRC_FP4 || srcfmt == SRC_FP4D;
        for (int tt = 0; tt < S.nh * nrb; ++tt, ++ti) {
          if (tt == 2 && !issue_next()) {
            ok = false;
            break;
          }
          const int i = tt / nrb, t = tt % nrb;
          const int rows = min(kFp4Rows, R - kFp4Rows * t);
          const size_t unit = (size_t)S.b * a.H + S.h0 + i;
          const size_t row_abs = unit * R + (size_t)kFp4Rows * t;  // first state row of the tile
          const uint32_t cs_bytes = srcfmt == SRC_FP4D ? (uint32_t)((rows + 15) / 16) * kCols : 0u;
          const int s = ti % NS;
          if (!mbar_wait_or_abort(&empty[s], (uint32_t)(((ti / NS) & 1) ^ 1), abort_flag, ws)) {
            ok = false;
            break;
          }
          unsigned char *st = stages + (size_t)s * lay.stage_bytes;
          const bool skp = (S.skip >> i) & 1u;  // decay-aware skip: no checkpoint tile for this head
          uint32_t tb = (uint32_t)n_rec * vrow;
          if (skp) {
          } else if (srcfmt == SRC_F32) tb += rows * kCols * 4;
          else if (srcfmt == SRC_F16) tb += rows * kCols * 2;
          else if (srcfmt == SRC_F8) tb += rows * kCols + 16;
          else tb += rows * (kCols / 2) + rows * (kCols / 16) + 16 + cs_bytes;
          if (lane == 0) {
            armed[s] = ti / NS;
            mbar_arrive_expect_tx(&full[s], tb);
          }
          __syncwarp();
          if (ti == a.withhold) continue;  // test hook: this stage is never filled
          if (lane == 0 && !skp) {
            if (srcfmt == SRC_F32)
              bulk_g2s(st, reinterpret_cast<const float *>(a.hp) + row_abs * kCols, rows * kCols * 4, &full[s], pol_stream);
            else if (srcfmt == SRC_F16)
              bulk_g2s(st, reinterpret_cast<const __half *>(a.hp) + row_abs * kCols, rows * kCols * 2, &full[s], pol_stream);
            else if (srcfmt == SRC_F8)
              bulk_g2s(st, static_cast<const unsigned char *>(a.hp) + row_abs * kCols, rows * kCols, &full[s], pol_stream);
            else
              bulk_g2s(st, a.rq + row_abs * (kCols / 2), rows * (kCols / 2), &full[s], pol_stream);
          }
          if (lane == 1 && fp4src && !skp) {
            bulk_g2s(st + kTileMaxBytes / 2, a.rs + row_abs * (kCols / 16), rows * (kCols / 16), &full[s], pol_stream);
            if (cs_bytes)
              bulk_g2s(st + kColScaleOff, a.rc + (unit * ((R + 15) / 16) + (size_t)t * (kFp4Rows / 16)) * kCols,
                       cs_bytes, &full[s], pol_stream);
          }
          if (lane == 2 && (fp4src || srcfmt == SRC_F8) && !skp) {
            const size_t gi4 = (unit * nrb + t) & ~(size_t)3;   // 16-byte chunk holding the tile scale
            bulk_g2s(st + lay.st_g, (fp4src ? a.rg : a.hs) + gi4, 16, &full[s], pol_keep);
          }
          if (lane == 3 && S.n_ring)
            bulk_g2s(st + lay.st_v, reinterpret_cast<const unsigned char *>(a.ring_v) + (unit * 2 * L + S.base_e) * vrow,
                     S.n_ring * vrow, &full[s], pol_keep);
          if (lane >= 4 && lane < 4 + S.n_new) {
            const int tk = lane - 4;
            bulk_g2s(st + lay.st_v + (S.n_ring + tk) * vrow,
                     reinterpret_cast<const unsigned char *>(a.v) + (((size_t)S.b * a.T + tk) * a.H + S.h0 + i) * vrow,
                     vrow, &full[s], pol_keep);
          }
        }
      }
      if (ok && !nxt_issued && !issue_next()) ok = false;
      if (!ok) break;
      Sc = Sn;
      u_cur = u_nxt;
      u_nxt = __shfl_sync(0xffffffffu, u_after, 0);
    }
    if (!ok && lane == 0) {
      record_error(a.err, 0, RSSM_DEV_TIMEOUT);
      *abort_flag = 1;
    }
  } else if (warp == kGPrep0 || warp == kGPrep0 + 1) {
    // ================================================================== prep warps
    const int pw = warp - kGPrep0;
    const int sg = pw * 4 + (lane >> 3), sl = lane & 7;       // 8 subgroups of 8 lanes
    const unsigned smask = 0xFFu << (lane & 24);
    int rdv = 0;  // rendezvous count (both prep warps take the same ones)
    auto prep_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(psync);
      const bool ok = mbar_wait_or_abort(psync, (uint32_t)(rdv & 1), abort_flag, ws);
      ++rdv;
      return ok;
    };
    for (int gi = 0;; ++gi) {
      const int gs = gi % kGBG, tsl = gi & 1;
      if (!mbar_wait_or_abort(&gfull[gs], (uint32_t)((gi / kGBG) & 1), abort_flag, ws) ||
          !mbar_wait_or_abort(&tempty[tsl], (uint32_t)(((gi >> 1) & 1) ^ 1), abort_flag, ws)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      if (gh[Q_END]) {  // no more units: let the consumers see the marker
        __syncwarp();
        if (pw == 0 && lane == 0) mbar_arrive(&tfull[tsl]);
        break;
      }
      float *gf = reinterpret_cast<float *>(gb);
      const int b = gh[Q_B], h0 = gh[Q_H0], nh = gh[Q_NH];
      if (pw == 0 && gh[Q_WMETA] && lane == 0) a.meta_out[b] = make_int4(gh[Q_MC], gh[Q_ME], gh[Q_MP], 0);
      const int active = gh[Q_ACTIVE];
      const int n_rec = gh[Q_NREC], m = gh[Q_M], n_ring = gh[Q_NRING], n_new = gh[Q_NNEW], t_out = gh[Q_TOUT];
      const int slot0 = gh[Q_SLOT0], base_e = gh[Q_BASE];
      const int kpe = lay.kpe != kCols && m > 0 ? lay.kpe : kCols;  // K row pitch of this unit (elements)
      if (active) {
        // alpha, beta of the new tokens (global loads) -> header; append k, alpha, beta to the ring
        for (int q = pw * 32 + lane; q < n_new * nh; q += 64) {
          const int t = q / nh, i = q % nh;
          const size_t tok = ((size_t)b * a.T + t) * a.H + h0 + i;
          const float al = a.alpha[tok], be = a.beta[tok];
          gf[Q_F + t * 8 + i] = al;
          gf[Q_FB + t * 8 + i] = be;
          const size_t unit = (size_t)b * a.H + h0 + i;
          a.ring_a[unit * dts + slot0 + t] = al;
          a.ring_b[unit * dts + slot0 + t] = be;
        }
        const int kq = kCols * esz / 16;
        for (int q = pw * 32 + lane; q < n_new * nh * kq; q += 64) {
          const int c16 = q % kq, ti2 = q / kq, t = ti2 / nh, i = ti2 % nh;
          const size_t unit = (size_t)b * a.H + h0 + i;
          const uint4 v = *reinterpret_cast<const uint4 *>(gb + lay.gb_k + ((size_t)i * lay.rmax + n_ring + t) * kpe * esz + c16 * 16);
          *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(a.ring_k) + ((unit * 2 * L + slot0 + t) * kCols) * esz +
                                     c16 * 16) = v;
        }
      }
      if (!prep_sync()) {  // both prep warps see the header floats
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      if (active && a.skip != nullptr && pw == 1 && lane < nh) {
        // skip flag for the next call: fp32 product of alpha, in record order, over the records
        // committed after this call (records m.. ; a verify's drafts are not committed)
        const int n_comm = a.op == OP_VERIFY ? n_ring : n_rec;
        const float *agf = reinterpret_cast<const float *>(gb + lay.gb_a);
        float prod = 1.f;
        for (int r = m; r < n_comm; ++r)
          prod = __fmul_rn(prod, r < n_ring ? agf[lane * dts + base_e + r] : gf[Q_F + (r - n_ring) * 8 + lane]);
        a.skip[(size_t)b * a.H + h0 + lane] = prod < a.skip_tau ? 1 : 0;
      }
      if (active) {
        float *u0t = reinterpret_cast<float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_u0);
        float *cot = reinterpret_cast<float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_coef);
        const TI *kg = reinterpret_cast<const TI *>(gb + lay.gb_k);
        const TI *qg = reinterpret_cast<const TI *>(gb + lay.gb_q);
        const float *ag = reinterpret_cast<const float *>(gb + lay.gb_a);
        const float *bg = reinterpret_cast<const float *>(gb + lay.gb_b);
        for (int p = sg; p < nh * t_out; p += 8) {
          const int i = p / t_out, j = p % t_out;
          const int e_j = n_rec - t_out + j + 1;
          float u[16];
          load_k16(qg + ((size_t)i * lay.no + j) * kCols + sl * 16, u);
          float *co = cot + ((size_t)i * lay.no + j) * lay.rmax;
          for (int r = sl; r < n_rec; r += 8)
            if (r < m || r >= e_j) co[r] = 0.f;
          // the walk-back is one dependent chain per (head, output): the next record's key and gates are
          // loaded while the current one is reduced, and the dot product runs as four partial sums
          auto gate = [&](int r, float &al, float &be) {
            al = r < n_ring ? ag[i * dts + base_e + r] : gf[Q_F + (r - n_ring) * 8 + i];
            be = r < n_ring ? bg[i * dts + base_e + r] : gf[Q_FB + (r - n_ring) * 8 + i];
          };
          float kn[16], aln = 0.f, ben = 0.f;
          if (e_j - 1 >= m) {
            load_k16(kg + ((size_t)i * lay.rmax + (e_j - 1)) * kpe + sl * 16, kn);
            gate(e_j - 1, aln, ben);
          }
          for (int r = e_j - 1; r >= m; --r) {
            float kv[16];
#pragma unroll
            for (int z = 0; z < 16; ++z) kv[z] = kn[z];
            const float al = aln, be = ben;
            if (r > m) {
              load_k16(kg + ((size_t)i * lay.rmax + (r - 1)) * kpe + sl * 16, kn);
              gate(r - 1, aln, ben);
            }
            float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
            for (int z = 0; z < 16; z += 4) {
              c0 = fmaf(u[z], kv[z], c0);
              c1 = fmaf(u[z + 1], kv[z + 1], c1);
              c2 = fmaf(u[z + 2], kv[z + 2], c2);
              c3 = fmaf(u[z + 3], kv[z + 3], c3);
            }
            float c = (c0 + c1) + (c2 + c3);
            c += __shfl_xor_sync(smask, c, 1);
            c += __shfl_xor_sync(smask, c, 2);
            c += __shfl_xor_sync(smask, c, 4);
            if (sl == 0) co[r] = a.q_scale * be * c;
            const float bc = be * c;
#pragma unroll
            for (int z = 0; z < 16; ++z) u[z] = al * fmaf(-bc, kv[z], u[z]);
          }
          float *ud = u0t + ((size_t)i * lay.no + j) * kCols + sl * 16;
          const float qs = a.q_scale;
#pragma unroll
          for (int z = 0; z < 16; z += 4)
            *reinterpret_cast<float4 *>(ud + z) = make_float4(qs * u[z], qs * u[z + 1], qs * u[z + 2], qs * u[z + 3]);
        }
      }
      if (active && m > 0) {  // per-record scalars of the fold: {alpha, beta, 1/alpha}
        float4 *abt = reinterpret_cast<float4 *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_ab);
        const float *ag = reinterpret_cast<const float *>(gb + lay.gb_a);
        const float *bg = reinterpret_cast<const float *>(gb + lay.gb_b);
        for (int q = pw * 32 + lane; q < nh * m; q += 64) {
          const int i = q / m, r = q % m;
          const float al = r < n_ring ? ag[i * dts + base_e + r] : gf[Q_F + (r - n_ring) * 8 + i];
          const float be = r < n_ring ? bg[i * dts + base_e + r] : gf[Q_FB + (r - n_ring) * 8 + i];
          abt[i * lay.rmax + r] = make_float4(al, be, __frcp_rn(al), 0.f);
        }
      }
      if (chunk && active && m > 0) {
        // chunked fold tables.  (1) The folded K rows (r < m) take the column order of the consumers' fragments:
        // in each 16-column chunk, columns {0,1,4,5,8,9,12,13} then {2,3,6,7,10,11,14,15} (bf16 pairs stay
        // together); the ring copies of the new rows were written above in the natural order, and the
        // walk-back reads only rows >= m.
        float *cht = reinterpret_cast<float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_ch);
        const int kpb = kpe * 2;
        for (int q = pw * 32 + lane; q < nh * m * 8; q += 64) {
          const int ih = q / (m * 8), rr = (q >> 3) % m, c = q & 7;
          uint4 *p = reinterpret_cast<uint4 *>(gb + lay.gb_k + ((size_t)ih * lay.rmax + rr) * kpb + c * 32);
          const uint4 w0 = p[0], w1 = p[1];
          p[0] = make_uint4(w0.x, w0.z, w1.x, w1.z);
          p[1] = make_uint4(w0.y, w0.w, w1.y, w1.w);
        }
        if (!prep_sync()) {  // K rows reordered
          if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
          break;
        }
        // (2) Per head (warp pw: heads pw, pw + 2), G = K K^T over the first 16 records on the tensor cores
        // (bf16 products exact, fp32 sums; rows past m repeat row m - 1): the ldmatrix fragments of K serve as
        // both operands.  The lane's accumulator entries (x, y) with x < y < m give
        // L_yx = beta_y (prod_{x<j<=y} alpha_j) G_xy, stored at T[y][x].
        const float *ag = reinterpret_cast<const float *>(gb + lay.gb_a);
        const float *bg = reinterpret_cast<const float *>(gb + lay.gb_b);
        auto alpha_of = [&](int ih, int r) { return r < n_ring ? ag[ih * dts + base_e + r] : gf[Q_F + (r - n_ring) * 8 + ih]; };
        const int gq = lane >> 2, tq = lane & 3;
        for (int ih = pw; ih < nh; ih += 2) {
          const unsigned char *kh = gb + lay.gb_k + ((size_t)ih * lay.rmax + min(lane & 15, m - 1)) * kpb + (lane >> 4) * 16;
          float g0[4] = {0.f, 0.f, 0.f, 0.f}, g1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < kCols / 16; ++ks) {
            uint32_t r0, r1, r2, r3;
            ldmatrix_x4(kh + ks * 32, r0, r1, r2, r3);
            mma_16816(g0, r0, r1, r2, r3, r0, r2);
            mma_16816(g1, r0, r1, r2, r3, r1, r3);
          }
          float al[kChMax];
#pragma unroll
          for (int j = 0; j < kChMax; ++j) al[j] = j < m ? alpha_of(ih, j) : 1.f;
          const float gv[8] = {g0[0], g0[1], g0[2], g0[3], g1[0], g1[1], g1[2], g1[3]};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int x = gq + 8 * ((q >> 1) & 1), y = 2 * tq + (q & 1) + 8 * (q >> 2);
            if (x < y && y < m) {
              float pf = y < n_ring ? bg[ih * dts + base_e + y] : gf[Q_FB + (y - n_ring) * 8 + ih];
#pragma unroll
              for (int j = 1; j < kChMax; ++j)
                if (j > x && j <= y) pf *= al[j];
              cht[ih * kChStride + y * kChMax + x] = pf * gv[q];
            }
          }
        }
        if (!prep_sync()) {  // L complete
          if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
          break;
        }
        // (3) T = (I + L)^-1 by forward substitution, lanes 0-15 and 16-31 one column each of two heads; the
        // whole 16 x 16 matrix is written (zero above the diagonal and past m), then a_r and b_r in record order
        for (int h2 = pw * 2; h2 < nh; h2 += 4) {
          const int ih = h2 + (lane >> 4), j = lane & 15;  // column j of head ih
          const bool hv = ih < nh;
          float *ch = cht + (hv ? ih : 0) * kChStride;
          float tcol[kChMax];  // T[r][j]
#pragma unroll
          for (int r = 0; r < kChMax; ++r) {
            float v = (r == j && j < m) ? 1.f : 0.f;
            if (hv && r > j && r < m) {
              float acc = 0.f;
#pragma unroll
              for (int i2 = 0; i2 < r; ++i2)
                if (i2 >= j) acc = fmaf(ch[r * kChMax + i2], tcol[i2], acc);
              v = -acc;
            }
            tcol[r] = v;
          }
          __syncwarp();  // every lane has read L before T overwrites it
          if (hv) {
#pragma unroll
            for (int r = 0; r < kChMax; ++r) ch[r * kChMax + j] = tcol[r];
            float ar = 0.f, br = 0.f;
            if (j < m) {
              ar = 1.f;
              br = 1.f;
              for (int jj = 0; jj <= j; ++jj) ar *= alpha_of(ih, jj);
              for (int jj = j + 1; jj < m; ++jj) br *= alpha_of(ih, jj);
            }
            ch[kChT + j] = ar;
            ch[kChT + kChMax + j] = br;
          }
          __syncwarp();
        }
      }
      if (!prep_sync()) {  // tables complete
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      if (pw == 0 && lane == 0) mbar_arrive(&tfull[tsl]);
    }
  } else {
    // ================================================================== consumer warps
    // All eight take every tile; warp w owns rows 8w..8w+7 of the 64-row tile.
    const int row0 = warp * 8;
    const uint64_t pol_wr = policy_evict_first();
    const uint64_t pol_ring = policy_evict_last();
    int ti = 0, rdv = 0, fd = 0;  // fd: fold tiles done (the two-axis copy's scratch slot rotates with it)
    int cft = 0;                  // chunked fold tiles seen (every consumer warp sees every tile)
    int crdv = 0;                 // rendezvous of this warp's group of four (chunked fold, NVFP4 copy)

    for (int gi = 0;; ++gi) {
      const int gs = gi % kGBG, tsl = gi & 1;
      if (!mbar_wait_or_abort(&tfull[tsl], (uint32_t)((gi >> 1) & 1), abort_flag, ws)) {
        if (lane == 0) { record_error(a.err, 0, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
        break;
      }
      const unsigned char *gb = gbuf + (size_t)gs * lay.gb_bytes;
      const int *gh = reinterpret_cast<const int *>(gb);
      if (gh[Q_END]) break;
      const int b = gh[Q_B], h0 = gh[Q_H0], nh = gh[Q_NH];
      if (gh[Q_ACTIVE]) {
        const int n_rec = gh[Q_NREC], m = gh[Q_M], t_out = gh[Q_TOUT];
        const int me = gh[Q_ME];
        const int n_ring = gh[Q_NRING], n_new = gh[Q_NNEW], slot0 = gh[Q_SLOT0];
        const unsigned skm = (unsigned)gh[Q_SKIP];
        const bool fold = m > 0;
        const int srcfmt = fold ? (shared_fp4 ? SRC_FP4 : hp_fmt)
                                : (fp4_read ? read_fmt : hp_fmt);
        const float *u0t = reinterpret_cast<const float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_u0);
        const float *cot = reinterpret_cast<const float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_coef);
        float *amx = reinterpret_cast<float *>(tabs + lay.tb_amax);  // [2 slots][8 warps], table buffer 0
        const TI *kg = reinterpret_cast<const TI *>(gb + lay.gb_k);
        for (int tt = 0; tt < nh * nrb; ++tt, ++ti) {
          const int i = tt / nrb, t = tt % nrb;
          const int rows = min(kFp4Rows, R - kFp4Rows * t);
          const int h = h0 + i;
          const size_t unit = (size_t)b * a.H + h;
          const int s = ti % NS;
          if (!mbar_wait_or_abort(&full[s], (uint32_t)((ti / NS) & 1), abort_flag, ws)) {
            if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
            break;
          }
          const unsigned char *st = stages + (size_t)s * lay.stage_bytes;
          const TI *vr = reinterpret_cast<const TI *>(st + lay.st_v);
          // the new tokens' v rows, landed behind the buffered ones in the head's first tile
          // stage, go to the head's ring row with one bulk store (warps take turns); every warp
          // waits for its bulk stores to have read the stage before releasing it
          // a chunked fold tile is taken by one group of four warps (alternating); the other group only
          // waits for it to land (so that its release cannot count for the stage's previous use) and releases it
          const bool gtile = fold && chunk;
          const int grp = cft & 1;
          cft += gtile ? 1 : 0;
          const bool mine = !gtile || (warp >> 2) == grp;
          const int vw = gtile ? 4 * grp + (ti & 3) : (ti & (kConsumerWarps - 1));
          if (t == 0 && n_new > 0 && vw == warp && lane == 0) {
            const uint32_t vrow = (uint32_t)R * esz;
            bulk_s2g(reinterpret_cast<unsigned char *>(a.ring_v) + (unit * 2 * a.L + slot0) * vrow,
                     st + lay.st_v + (size_t)n_ring * vrow, (uint32_t)n_new * vrow, pol_ring);
            bulk_commit();
          }
          const float g_tile = reinterpret_cast<const float *>(st + lay.st_g)[(unit * nrb + t) & 3];
          const float *co_h = cot + (size_t)i * lay.no * lay.rmax;
          const float *u0_h = u0t + (size_t)i * lay.no * kCols;
          // 4 consecutive state values of tile row `row` starting at column `col`, from the stage
          auto load_row4 = [&](int row, int col) -> float4 {
            if (srcfmt == SRC_F32) return *reinterpret_cast<const float4 *>(st + (row * kCols + col) * 4);
            if (srcfmt == SRC_F16) {
              const uint2 hv = *reinterpret_cast<const uint2 *>(st + (row * kCols + col) * 2);
              const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&hv.x));
              const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&hv.y));
              return make_float4(f0.x, f0.y, f1.x, f1.y);
            }
            if (srcfmt == SRC_F8) {  // E4M3 codes times the tile scale
              const float4 e = e4m3x4_to_float4(*reinterpret_cast<const uint32_t *>(st + row * kCols + col));
              return make_float4(__fmul_rn(e.x, g_tile), __fmul_rn(e.y, g_tile), __fmul_rn(e.z, g_tile),
                                 __fmul_rn(e.w, g_tile));
            }
            // NVFP4: E2M1 codes times the block step d_b = E4M3 block scale times the tile scale (two-axis
            // copy: times 2^-8; its column-group step is applied to the vector the row is multiplied with)
            const uint32_t cw = *reinterpret_cast<const uint16_t *>(st + row * (kCols / 2) + col / 2);
            const uint32_t sc = st[kTileMaxBytes / 2 + row * (kCols / 16) + col / 16];
            const float d_b = __fmul_rn(e4m3_to_float(sc), srcfmt == SRC_FP4D ? 0.00390625f : g_tile);
            const float4 e = e2m1x4_to_float4(cw);
            return make_float4(__fmul_rn(e.x, d_b), __fmul_rn(e.y, d_b), __fmul_rn(e.z, d_b), __fmul_rn(e.w, d_b));
          };
          if (!mine) {
          } else if (!fold) {
            // ---------------- non-fold tile: lane owns columns 4l..4l+3 of the warp's 8 rows
            if (row0 < rows) {
              constexpr int V = 8 * NO;
              constexpr int KEEP = V >= 32 ? V / 32 : 1;
              constexpr int SPREAD = V >= 32 ? 1 : 32 / V;
              float4 uv[NO];
#pragma unroll
              for (int j = 0; j < NO; ++j)
                uv[j] = (j < t_out) ? *reinterpret_cast<const float4 *>(u0_h + j * kCols + 4 * lane) : make_float4(0, 0, 0, 0);
              if (srcfmt == SRC_FP4D) {  // column-group steps k = E4M3 * g of this warp's 16-row group
                const float4 c4 = e4m3x4_to_float4(
                    *reinterpret_cast<const uint32_t *>(st + kColScaleOff + (row0 >> 4) * kCols + 4 * lane));
                const float4 k4 = make_float4(__fmul_rn(c4.x, g_tile), __fmul_rn(c4.y, g_tile), __fmul_rn(c4.z, g_tile),
                                              __fmul_rn(c4.w, g_tile));
#pragma unroll
                for (int j = 0; j < NO; ++j) {
                  uv[j].x *= k4.x; uv[j].y *= k4.y; uv[j].z *= k4.z; uv[j].w *= k4.w;
                }
              }
              float4 sv[8];
              float dstep[8];  // NVFP4 copies: the row's block step, applied to the row's dot product
#pragma unroll
              for (int rr = 0; rr < 8; ++rr) dstep[rr] = 1.f;
              if ((skm >> i) & 1u) {  // skipped head: the checkpoint term is zero
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) sv[rr] = make_float4(0.f, 0.f, 0.f, 0.f);
              } else if (srcfmt == SRC_F32) {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr)
                  sv[rr] = *reinterpret_cast<const float4 *>(st + ((row0 + rr) * kCols + 4 * lane) * 4);
              } else if (srcfmt == SRC_FP4 || srcfmt == SRC_FP4D) {
                // the lane's 4 columns lie in one 16-element block of each row: E2M1 values here, the block
                // step once per row
                const float dmul = srcfmt == SRC_FP4D ? 0.00390625f : g_tile;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                  const int row = row0 + rr;
                  sv[rr] = e2m1x4_to_float4(*reinterpret_cast<const uint16_t *>(st + row * (kCols / 2) + 2 * lane));
                  dstep[rr] = __fmul_rn(e4m3_to_float(st[kTileMaxBytes / 2 + row * (kCols / 16) + (lane >> 2)]), dmul);
                }
              } else {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) sv[rr] = load_row4(row0 + rr, 4 * lane);
              }
              float part[V];
#pragma unroll
              for (int rr = 0; rr < 8; ++rr)
#pragma unroll
                for (int j = 0; j < NO; ++j)
                  part[rr * NO + j] =
                      dstep[rr] * (sv[rr].x * uv[j].x + sv[rr].y * uv[j].y + sv[rr].z * uv[j].z + sv[rr].w * uv[j].w);
              // buffered part: lane r adds coef_{j,r} v_r[row] for the 8 rows (one 16-byte load of v_r)
              for (int r = lane; r < n_rec; r += 32) {
                float vv[8];
                load8(vr + r * R + kFp4Rows * t + row0, vv);
#pragma unroll
                for (int j = 0; j < NO; ++j) {
                  const float co = (j < t_out) ? co_h[j * lay.rmax + r] : 0.f;
#pragma unroll
                  for (int rr = 0; rr < 8; ++rr) part[rr * NO + j] = fmaf(co, vv[rr], part[rr * NO + j]);
                }
              }
              warp_transpose_reduce<V>(part, lane);
#pragma unroll
              for (int k2 = 0; k2 < KEEP; ++k2) {
                const int idx = (V >= 32) ? lane * KEEP + k2 : lane / SPREAD;
                const int rr = idx / NO, j = idx % NO;
                if (j < t_out && (lane % SPREAD) == 0)
                  a.y[(((size_t)b * a.T + j) * a.H + h) * R + kFp4Rows * t + row0 + rr] = part[k2];
              }
            }
          } else if (chunk) {
            // ---------------- chunked fold tile: warp (w & 3) of the group owns rows 16(w & 3) .. +15 and computes
            // their new state alone.  Lane 4g+t holds rows ra = 16(w & 3) + g and rb = ra + 8, and in each
            // 16-column chunk c the columns 16c + 4t .. +3, which the reordered K rows match as fragments.
            const float *cht = reinterpret_cast<const float *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_ch) +
                               i * kChStride;
            const float4 *abt = reinterpret_cast<const float4 *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_ab) +
                                (size_t)i * lay.rmax;
            const int kpb = lay.kpe * 2;  // K row pitch in bytes (bf16)
            const unsigned char *kb = gb + lay.gb_k + (size_t)i * lay.rmax * kpb;
            unsigned char *stw = stages + (size_t)s * lay.stage_bytes;
            const int gq = lane >> 2, qtr = lane & 3, odd = gq & 1;
            const int wr0 = 16 * (warp & 3), ra = wr0 + gq, rb = ra + 8;
            const bool va = ra < rows, vb = rb < rows;
            const bool skp = (skm >> i) & 1u;  // a skipped head folds from zero
            const bool la = va && !skp, lb = vb && !skp;
            const int rga = kFp4Rows * t + ra, rgb = rga + 8;  // rows within the head's state
            auto srow = [&](int r, int c) { return reinterpret_cast<float4 *>(stw + ((size_t)r * kCols + 16 * c + 4 * qtr) * 4); };
            // chunks cp and cp + 1 of rows ra, rb from the stage; rows of odd g take the pair in the other order,
            // so that the loads (and the stores back) are free of bank conflicts
            auto load_pair = [&](int cp, float4 (&xa)[2], float4 (&xb)[2]) {
              const int c0 = cp + odd, c1 = cp + 1 - odd;
              const float4 pa = la ? *srow(ra, c0) : f4zero(), pb = lb ? *srow(rb, c0) : f4zero();
              const float4 qa = la ? *srow(ra, c1) : f4zero(), qb = lb ? *srow(rb, c1) : f4zero();
              xa[0] = odd ? qa : pa; xa[1] = odd ? pa : qa;
              xb[0] = odd ? qb : pb; xb[1] = odd ? pb : qb;
            };
            // phase 1: Z = S K^T for records 0-7 and 8-15 (rows past m repeat row m - 1; their columns of Z are
            // not used) in tf32: per 16-column chunk two k-steps of 8 (lane t's columns 4t, 4t+1, then 4t+2,
            // 4t+3), S in two tf32 pieces (hi: the leading 11 bits, lo: the next 11, so |s - hi - lo| < 2^-20 |s|),
            // K exact (a bf16 widened); the small pieces first.  Where the fold result is re-quantised (the
            // NVFP4 copy), S takes three pieces (the third holds the last 2 bits, so the sum is exact): Z then
            // carries no representation error, and the copy's decisions follow the fp32 result more closely.
            constexpr bool kZ3 = LP;
            float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
            const bool two = m > 8;
            const unsigned char *kl = kb + (size_t)min((lane & 7) + 8 * (lane >> 4), m - 1) * kpb + ((lane >> 3) & 1) * 16;
            auto tf32_split = [](float x, uint32_t &hi, uint32_t &lo, uint32_t &lo2) {
              hi = __float_as_uint(x) & 0xffffe000u;
              const float r = x - __uint_as_float(hi);
              lo = __float_as_uint(r) & 0xffffe000u;
              lo2 = kZ3 ? __float_as_uint(r - __uint_as_float(lo)) : 0u;
            };
#pragma unroll
            for (int cp = 0; cp < 8; cp += 2) {
              float4 xa[2], xb[2];
              load_pair(cp, xa, xb);
#pragma unroll
              for (int o = 0; o < 2; ++o) {
                uint32_t q0, q1, q2, q3;  // records 0-7: columns (4t, 4t+1) in q0, (4t+2, 4t+3) in q1; 8-15: q2, q3
                ldmatrix_x4(kl + (cp + o) * 32, q0, q1, q2, q3);
                uint32_t ah[2][4], al[2][4], a3[2][4];  // [k-step][fragment register]
                tf32_split(xa[o].x, ah[0][0], al[0][0], a3[0][0]); tf32_split(xb[o].x, ah[0][1], al[0][1], a3[0][1]);
                tf32_split(xa[o].y, ah[0][2], al[0][2], a3[0][2]); tf32_split(xb[o].y, ah[0][3], al[0][3], a3[0][3]);
                tf32_split(xa[o].z, ah[1][0], al[1][0], a3[1][0]); tf32_split(xb[o].z, ah[1][1], al[1][1], a3[1][1]);
                tf32_split(xa[o].w, ah[1][2], al[1][2], a3[1][2]); tf32_split(xb[o].w, ah[1][3], al[1][3], a3[1][3]);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                  const uint32_t w0 = kk ? q1 : q0, w1 = kk ? q3 : q2;
                  if (kZ3) mma_1688_tf32(z0, a3[kk][0], a3[kk][1], a3[kk][2], a3[kk][3], w0 << 16, w0 & 0xffff0000u);
                  mma_1688_tf32(z0, al[kk][0], al[kk][1], al[kk][2], al[kk][3], w0 << 16, w0 & 0xffff0000u);
                  mma_1688_tf32(z0, ah[kk][0], ah[kk][1], ah[kk][2], ah[kk][3], w0 << 16, w0 & 0xffff0000u);
                  if (two) {
                    if (kZ3) mma_1688_tf32(z1, a3[kk][0], a3[kk][1], a3[kk][2], a3[kk][3], w1 << 16, w1 & 0xffff0000u);
                    mma_1688_tf32(z1, al[kk][0], al[kk][1], al[kk][2], al[kk][3], w1 << 16, w1 & 0xffff0000u);
                    mma_1688_tf32(z1, ah[kk][0], ah[kk][1], ah[kk][2], ah[kk][3], w1 << 16, w1 & 0xffff0000u);
                  }
                }
              }
            }
            // phase 2: rt_r = beta_r (v_r[row] - a_r z_r) for the lane's records 2t, 2t+1, 2t+8, 2t+9 (zero past
            // m), then U = RT T^T on the tensor cores (both fp32 operands in three pieces; the six piece
            // products above 2^-24 kept): U lands on the lane's own records, as the A operand of phase 3 wants
            float rta[4], rtb[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int r = 2 * qtr + (k & 1) + 8 * (k >> 1);
              const float za = k < 2 ? z0[k & 1] : z1[k & 1];
              const float zb = k < 2 ? z0[2 + (k & 1)] : z1[2 + (k & 1)];
              float xa = 0.f, xb = 0.f;
              if (r < m) {
                const float be = abt[r].y, ar = cht[kChT + r];
                xa = be * ((va ? to_f32(vr[r * R + rga]) : 0.f) - ar * za);
                xb = be * ((vb ? to_f32(vr[r * R + rgb]) : 0.f) - ar * zb);
              }
              rta[k] = xa;
              rtb[k] = xb;
            }
            float wa[4], wb[4];
            {
              uint32_t rp[3][4];
              split3_bf16x2(rta[0], rta[1], rp[0][0], rp[1][0], rp[2][0]);
              split3_bf16x2(rtb[0], rtb[1], rp[0][1], rp[1][1], rp[2][1]);
              split3_bf16x2(rta[2], rta[3], rp[0][2], rp[1][2], rp[2][2]);
              split3_bf16x2(rtb[2], rtb[3], rp[0][3], rp[1][3], rp[2][3]);
              float u[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
              for (int nt = 0; nt < 2; ++nt) {
                const float *tr = cht + (8 * nt + gq) * kChMax + 2 * qtr;  // B[i][r] = T[r][i], r = 8nt + g
                const float2 t0 = *reinterpret_cast<const float2 *>(tr), t1 = *reinterpret_cast<const float2 *>(tr + 8);
                uint32_t tp0[3], tp1[3];
                split3_bf16x2(t0.x, t0.y, tp0[0], tp0[1], tp0[2]);
                split3_bf16x2(t1.x, t1.y, tp1[0], tp1[1], tp1[2]);
                constexpr int kPa[6] = {2, 1, 0, 1, 0, 0}, kPb[6] = {0, 1, 2, 0, 1, 0};
#pragma unroll
                for (int q = 0; q < 6; ++q)
                  mma_16816(u[nt], rp[kPa[q]][0], rp[kPa[q]][1], rp[kPa[q]][2], rp[kPa[q]][3], tp0[kPb[q]], tp1[kPb[q]]);
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int r = 2 * qtr + (k & 1) + 8 * (k >> 1);
                const float br = cht[kChT + kChMax + r];  // zero past m
                wa[k] = br * u[k >> 1][k & 1];
                wb[k] = br * u[k >> 1][2 + (k & 1)];
              }
            }
            // phase 3: S' = a_{m-1} S + W K over 16 n-tiles: B from the reordered K rows with ldmatrix.trans
            // (records past m masked to zero), D on the lane's own columns
            uint32_t wp[3][4];
            split3_bf16x2(wa[0], wa[1], wp[0][0], wp[1][0], wp[2][0]);
            split3_bf16x2(wb[0], wb[1], wp[0][1], wp[1][1], wp[2][1]);
            split3_bf16x2(wa[2], wa[3], wp[0][2], wp[1][2], wp[2][2]);
            split3_bf16x2(wb[2], wb[3], wp[0][3], wp[1][3], wp[2][3]);
            const float am = cht[kChT + m - 1];
            const uint32_t mk0 = (2 * qtr < m ? 0xFFFFu : 0u) | (2 * qtr + 1 < m ? 0xFFFF0000u : 0u);
            const uint32_t mk1 = (2 * qtr + 8 < m ? 0xFFFFu : 0u) | (2 * qtr + 9 < m ? 0xFFFF0000u : 0u);
            const unsigned char *kt = kb + (size_t)min((lane & 7) + 8 * ((lane >> 3) & 1), m - 1) * kpb + (lane >> 4) * 16;
            // S is read again from the stage chunk pair by chunk pair, and S' goes back to the same place
            float smax = 0.f;  // the largest magnitude of the lane's rows of S' (NVFP4 copy: the tile scale)
#pragma unroll
            for (int cp = 0; cp < 8; cp += 2) {
              float4 xa[2], xb[2];
              load_pair(cp, xa, xb);
#pragma unroll
              for (int o2 = 0; o2 < 2; ++o2) {
                const int c = cp + o2;
                uint32_t q0, q1, q2, q3;  // n-tile (c, 0): q0 (records 0-7), q1 (8-15); n-tile (c, 1): q2, q3
                ldmatrix_x4_trans(kt + c * 32, q0, q1, q2, q3);
#pragma unroll
                for (int o = 0; o < 2; ++o) {
                  const uint32_t b0 = (o ? q2 : q0) & mk0, b1 = (o ? q3 : q1) & mk1;
                  float d[4];
                  if (o == 0) { d[0] = xa[o2].x * am; d[1] = xa[o2].y * am; d[2] = xb[o2].x * am; d[3] = xb[o2].y * am; }
                  else        { d[0] = xa[o2].z * am; d[1] = xa[o2].w * am; d[2] = xb[o2].z * am; d[3] = xb[o2].w * am; }
#pragma unroll
                  for (int p = 2; p >= 0; --p) mma_16816(d, wp[p][0], wp[p][1], wp[p][2], wp[p][3], b0, b1);
                  if (o == 0) { xa[o2].x = d[0]; xa[o2].y = d[1]; xb[o2].x = d[2]; xb[o2].y = d[3]; }
                  else        { xa[o2].z = d[0]; xa[o2].w = d[1]; xb[o2].z = d[2]; xb[o2].w = d[3]; }
                }
                if (fp4_read) {
                  if (va) smax = fmaxf(smax, fmaxf(fmaxf(fabsf(xa[o2].x), fabsf(xa[o2].y)), fmaxf(fabsf(xa[o2].z), fabsf(xa[o2].w))));
                  if (vb) smax = fmaxf(smax, fmaxf(fmaxf(fabsf(xb[o2].x), fabsf(xb[o2].y)), fmaxf(fabsf(xb[o2].z), fabsf(xb[o2].w))));
                }
              }
              const int c0 = cp + odd, c1 = cp + 1 - odd;
              *srow(ra, c0) = odd ? xa[1] : xa[0];
              *srow(rb, c0) = odd ? xb[1] : xb[0];
              *srow(ra, c1) = odd ? xa[0] : xa[1];
              *srow(rb, c1) = odd ? xb[0] : xb[1];
            }
            // the outputs from S' (each lane reads back what it wrote; u_0 carries q_scale), the buffered
            // records past the fold, then the quad's partial sums
            for (int j = 0; j < t_out; ++j) {
              const int e_j = n_rec - t_out + j + 1;
              float ya = 0.f, yb = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int cc = c ^ odd;  // odd rows in the other chunk order, as written
                const float4 u = *reinterpret_cast<const float4 *>(u0_h + j * kCols + 16 * cc + 4 * qtr);
                const float4 sa = *srow(ra, cc), sb = *srow(rb, cc);
                ya = fmaf(sa.x, u.x, fmaf(sa.y, u.y, fmaf(sa.z, u.z, fmaf(sa.w, u.w, ya))));
                yb = fmaf(sb.x, u.x, fmaf(sb.y, u.y, fmaf(sb.z, u.z, fmaf(sb.w, u.w, yb))));
              }
              for (int r = m + qtr; r < e_j; r += 4) {
                const float co = co_h[j * lay.rmax + r];
                if (va) ya = fmaf(co, to_f32(vr[r * R + rga]), ya);
                if (vb) yb = fmaf(co, to_f32(vr[r * R + rgb]), yb);
              }
              ya += __shfl_xor_sync(0xffffffffu, ya, 1);
              yb += __shfl_xor_sync(0xffffffffu, yb, 1);
              ya += __shfl_xor_sync(0xffffffffu, ya, 2);
              yb += __shfl_xor_sync(0xffffffffu, yb, 2);
              float *yj = a.y + (((size_t)b * a.T + j) * a.H + h) * R;
              if (qtr == 0 && va) yj[rga] = ya;
              if (qtr == 0 && vb) yj[rgb] = yb;
            }
            fence_async_smem();
            __syncwarp();
            const int wrows = min(16, rows - wr0);
            if (lane == 0 && wrows > 0) {
              bulk_s2g(static_cast<unsigned char *>(a.hp) + (unit * R + kFp4Rows * t + wr0) * kCols * 4,
                       stw + (size_t)wr0 * kCols * 4, (uint32_t)(wrows * kCols * 4), pol_wr);
              bulk_commit();
            }
            if (fp4_read) {
              // the NVFP4 read copy of S': the tile scale from the maximum over the group's four warps (their
              // rendezvous through an mbarrier with bounded waits), then per row the block scales and codes,
              // chunk c of a row being its block c (the quad's four lanes share a block)
              float wmx = smax;
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1) wmx = fmaxf(wmx, __shfl_xor_sync(0xffffffffu, wmx, off));
              float *gmx = amx + grp * 8 + (crdv & 1) * 4;  // [group][slot][warp of the group]
              if (lane == 0) gmx[warp & 3] = wmx;
              __syncwarp();
              if (lane == 0) mbar_arrive(&csync[grp]);
              if (!mbar_wait_or_abort(&csync[grp], (uint32_t)(crdv & 1), abort_flag, ws)) {
                if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
                break;
              }
              ++crdv;
              const float g = nvfp4_tile_scale(fmaxf(fmaxf(gmx[0], gmx[1]), fmaxf(gmx[2], gmx[3])));
              if ((warp & 3) == 0 && lane == 0) a.rg[unit * nrb + t] = g;
              // the quad's 16 (row, block) pairs p = 8 hr + c (row ra or rb, chunk slot c, block c ^ odd): their
              // maxima by a transposing reduction over the quad, after which lane qtr holds the pairs
              // 8 b0 + 4 b1 + k (b0 = qtr & 1, b1 = qtr >> 1) and computes their scales once; the steps and
              // their reciprocals then travel back to every lane of the quad
              const bool b0 = qtr & 1, b1 = (qtr >> 1) & 1;
              float bmx[16];
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float4 pa = va ? *srow(ra, c ^ odd) : f4zero(), pb = vb ? *srow(rb, c ^ odd) : f4zero();
                bmx[c] = fmaxf(fmaxf(fabsf(pa.x), fabsf(pa.y)), fmaxf(fabsf(pa.z), fabsf(pa.w)));
                bmx[8 + c] = fmaxf(fmaxf(fabsf(pb.x), fabsf(pb.y)), fmaxf(fabsf(pb.z), fabsf(pb.w)));
              }
              float w8[8], w4[4];
#pragma unroll
              for (int k = 0; k < 8; ++k)
                w8[k] = fmaxf(b0 ? bmx[k + 8] : bmx[k], __shfl_xor_sync(0xffffffffu, b0 ? bmx[k] : bmx[k + 8], 1));
#pragma unroll
              for (int k = 0; k < 4; ++k)
                w4[k] = fmaxf(b1 ? w8[k + 4] : w8[k], __shfl_xor_sync(0xffffffffu, b1 ? w8[k] : w8[k + 4], 2));
              float dq[4], rq[4];
              uint32_t scw = 0u;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                scw |= nvfp4_block_scale(w4[k], g, &dq[k]) << (8 * (k ^ odd));
                rq[k] = __frcp_rn(dq[k]);
              }
              if (b0 ? vb : va)  // row rb (b0) or ra, blocks 4 b1 .. 4 b1 + 3
                *reinterpret_cast<uint32_t *>(a.rs + (unit * R + (b0 ? rgb : rga)) * (kCols / 16) + 4 * b1) = scw;
              float d8[8], r8[8], d16[16], r16[16];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float od = __shfl_xor_sync(0xffffffffu, dq[k], 2), orr = __shfl_xor_sync(0xffffffffu, rq[k], 2);
                d8[k] = b1 ? od : dq[k]; d8[k + 4] = b1 ? dq[k] : od;
                r8[k] = b1 ? orr : rq[k]; r8[k + 4] = b1 ? rq[k] : orr;
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float od = __shfl_xor_sync(0xffffffffu, d8[k], 1), orr = __shfl_xor_sync(0xffffffffu, r8[k], 1);
                d16[k] = b0 ? od : d8[k]; d16[k + 8] = b0 ? d8[k] : od;
                r16[k] = b0 ? orr : r8[k]; r16[k + 8] = b0 ? r8[k] : orr;
              }
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int cc = c ^ odd;
                if (va) {
                  const uint32_t cw = nvfp4_code4(*srow(ra, cc), d16[c], r16[c]);
                  *reinterpret_cast<uint16_t *>(a.rq + (unit * R + rga) * (kCols / 2) + cc * 8 + qtr * 2) = (uint16_t)cw;
                }
                if (vb) {
                  const uint32_t cw = nvfp4_code4(*srow(rb, cc), d16[8 + c], r16[8 + c]);
                  *reinterpret_cast<uint16_t *>(a.rq + (unit * R + rgb) * (kCols / 2) + cc * 8 + qtr * 2) = (uint16_t)cw;
                }
              }
            }
          } else {
            // ---------------- fold tile: four lanes per row, 32 columns each, chunks rotated by lane
            const int qtr = lane & 3;
            const int row = row0 + (lane >> 2);
            const bool live = row < rows;
            const int rowg = kFp4Rows * t + row;  // row within the head's state
            const bool from_ckpt = live && !((skm >> i) & 1u);  // a skipped head folds from zero
            float4 sv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int ch = (c + lane) & 7;
              sv[c] = from_ckpt ? load_row4(row, qtr * 32 + ch * 4) : make_float4(0, 0, 0, 0);
            }
            // s <- alpha s + beta (v[row] - alpha (s . k)) k, record by record.  The row is kept as
            // s = sig * s~ so that each record costs one FMA per element: s~ += (coef / sig') k with
            // sig' = alpha sig, and s . k = sig (s~ . k); s~ is rescaled if sig gets small.
            float sig = 1.f, isig = 1.f;
            const float4 *abt = reinterpret_cast<const float4 *>(tabs + (size_t)tsl * lay.tab_bytes + lay.tb_ab) +
                                (size_t)i * lay.rmax;
            for (int r = 0; r < m; ++r) {
              const TI *kr = kg + ((size_t)i * lay.rmax + r) * lay.kpe + qtr * 32;
              float4 kv[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) kv[c] = load4(kr + ((c + lane) & 7) * 4);
              const float4 abr = abt[r];
              const float al = abr.x, be = abr.y;
              const float vrow = live ? to_f32(vr[r * R + rowg]) : 0.f;
              float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                d0 = fmaf(sv[c].x, kv[c].x, d0);
                d1 = fmaf(sv[c].y, kv[c].y, d1);
                d2 = fmaf(sv[c].z, kv[c].z, d2);
                d3 = fmaf(sv[c].w, kv[c].w, d3);
              }
              float d = (d0 + d1) + (d2 + d3);
              d += __shfl_xor_sync(0xffffffffu, d, 1);
              d += __shfl_xor_sync(0xffffffffu, d, 2);
              const float coef = be * (vrow - al * (sig * d));
              sig *= al;
              isig *= abr.z;
              if (sig < 9.3e-10f) {  // 2^-30: fold the scale back into the row
#pragma unroll
                for (int c = 0; c < 8; ++c) { sv[c].x *= sig; sv[c].y *= sig; sv[c].z *= sig; sv[c].w *= sig; }
                sig = 1.f;
                isig = 1.f;
              }
              const float cs = coef * isig;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                sv[c].x = fmaf(cs, kv[c].x, sv[c].x);
                sv[c].y = fmaf(cs, kv[c].y, sv[c].y);
                sv[c].z = fmaf(cs, kv[c].z, sv[c].z);
                sv[c].w = fmaf(cs, kv[c].w, sv[c].w);
              }
            }
            if (sig != 1.f) {
#pragma unroll
              for (int c = 0; c < 8; ++c) { sv[c].x *= sig; sv[c].y *= sig; sv[c].z *= sig; sv[c].w *= sig; }
            }
            // outputs from the fp32 fold result (u_0 and the coefficients carry q_scale)
            for (int j = 0; j < t_out; ++j) {
              const float *uj = u0_h + j * kCols + qtr * 32;
              float z = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float4 uv = *reinterpret_cast<const float4 *>(uj + ((c + lane) & 7) * 4);
                z = fmaf(sv[c].x, uv.x, fmaf(sv[c].y, uv.y, fmaf(sv[c].z, uv.z, fmaf(sv[c].w, uv.w, z))));
              }
              const int e_j = n_rec - t_out + j + 1;
              if (live)
                for (int r = m + qtr; r < e_j; r += 4) z = fmaf(co_h[j * lay.rmax + r], to_f32(vr[r * R + rowg]), z);
              z += __shfl_xor_sync(0xffffffffu, z, 1);
              z += __shfl_xor_sync(0xffffffffu, z, 2);
              if (live && qtr == 0) a.y[(((size_t)b * a.T + j) * a.H + h) * R + rowg] = z;
            }
            // the E4M3 checkpoint and the NVFP4 read copy both scale by the maximum over the
            // 64-row tile, which spans the eight warps: each posts its rows' maximum, then all read them
            float tmax = 0.f;
            if (fp4_read || hp8) {
              float am = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                am = fmaxf(am, fmaxf(fmaxf(fabsf(sv[c].x), fabsf(sv[c].y)), fmaxf(fabsf(sv[c].z), fabsf(sv[c].w))));
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
              const int slot = rdv & 1;
              if (lane == 0) amx[slot * 8 + warp] = am;
              if (fp4d) {
                // two-axis copy: column maxima of each 16-row group into this tile's slot, and the slot of the
                // fold tile after next cleared (every warp has read it before the previous rendezvous)
                unsigned int *cm = cmx + (fd % 3) * kCmSlotWords + (row >> 4) * kCols + qtr * 32;
                if (live) {
#pragma unroll
                  for (int c = 0; c < 8; ++c) {
                    unsigned int *cc = cm + ((c + lane) & 7) * 4;
                    atomicMax(cc, __float_as_uint(fabsf(sv[c].x)));
                    atomicMax(cc + 1, __float_as_uint(fabsf(sv[c].y)));
                    atomicMax(cc + 2, __float_as_uint(fabsf(sv[c].z)));
                    atomicMax(cc + 3, __float_as_uint(fabsf(sv[c].w)));
                  }
                }
                unsigned int *cz = cmx + ((fd + 1) % 3) * kCmSlotWords;
                for (int q = warp * 32 + lane; q < kCmSlotWords; q += kConsumers) cz[q] = 0u;
                __threadfence_block();
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(fsync);  // every consumer warp has posted its maximum
              if (!mbar_wait_or_abort(fsync, (uint32_t)(rdv & 1), abort_flag, ws)) {
                if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
                break;
              }
              ++rdv;
#pragma unroll
              for (int w = 0; w < kConsumerWarps; ++w) tmax = fmaxf(tmax, amx[slot * 8 + w]);
              if (fp4d) {
                // the column-group steps k = E4M3 * g (two per thread) and their codes; every warp reads the
                // steps after a second rendezvous
                const unsigned int *cm = cmx + (fd % 3) * kCmSlotWords;
                const float g = nvfp4_tile_scale(tmax);
                unsigned char *rcd = a.rc + (unit * ((R + 15) / 16) + (size_t)t * (kFp4Rows / 16)) * kCols;
                for (int q = warp * 32 + lane; q < ((rows + 15) >> 4) * kCols; q += kConsumers) {
                  float k;
                  rcd[q] = (unsigned char)nvfp4d_col_scale(__uint_as_float(cm[q]), g, &k);
                  kvals[q] = k;
                }
                ++fd;
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(fsync);
                if (!mbar_wait_or_abort(fsync, (uint32_t)(rdv & 1), abort_flag, ws)) {
                  if (lane == 0) { record_error(a.err, b, RSSM_DEV_TIMEOUT); *abort_flag = 1; }
                  break;
                }
                ++rdv;
              }
            }
            // write the new state in the checkpoint format: each lane puts its values back where it
            // read them in the stage, then one bulk store per warp moves the warp's rows (contiguous
            // in shared and in global memory) with full-line writes
            if (!shared_fp4) {
              unsigned char *stw = stages + (size_t)s * lay.stage_bytes;
              const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32);
              const float s8 = fp8_tile_scale(tmax);
              if (live) {
                if (hp_fmt == SRC_F32) {
#pragma unroll
                  for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4 *>(stw + (row * kCols + qtr * 32 + ((c + lane) & 7) * 4) * 4) = sv[c];
                } else if (hp16) {
#pragma unroll
                  for (int c = 0; c < 8; ++c) {
                    const int ch = (c + lane) & 7;
                    const uint32_t elem = (uint32_t)(rowg * kCols + qtr * 32 + ch * 4);
                    const uint4 rw = philox4x32_10(make_uint4((uint32_t)unit, (uint32_t)me, elem >> 2, 0u), k0, k1);
                    const __half h0v = fp16_sr(sv[c].x, rw.x), h1v = fp16_sr(sv[c].y, rw.y);
                    const __half h2v = fp16_sr(sv[c].z, rw.z), h3v = fp16_sr(sv[c].w, rw.w);
                    uint2 pk;
                    pk.x = (uint32_t)__half_as_ushort(h0v) | ((uint32_t)__half_as_ushort(h1v) << 16);
                    pk.y = (uint32_t)__half_as_ushort(h2v) | ((uint32_t)__half_as_ushort(h3v) << 16);
                    *reinterpret_cast<uint2 *>(stw + (row * kCols + qtr * 32 + ch * 4) * 2) = pk;
                  }
                } else {
#pragma unroll
                  for (int c = 0; c < 8; ++c) {
                    const int ch = (c + lane) & 7;
                    const uint32_t elem = (uint32_t)(rowg * kCols + qtr * 32 + ch * 4);
                    const uint4 rw = philox4x32_10(make_uint4((uint32_t)unit, (uint32_t)me, elem >> 2, 0u), k0, k1);
                    const uint32_t pk = fp8_sr_code(__fdiv_rn(sv[c].x, s8), rw.x) |
                                        (fp8_sr_code(__fdiv_rn(sv[c].y, s8), rw.y) << 8) |
                                        (fp8_sr_code(__fdiv_rn(sv[c].z, s8), rw.z) << 16) |
                                        (fp8_sr_code(__fdiv_rn(sv[c].w, s8), rw.w) << 24);
                    *reinterpret_cast<uint32_t *>(stw + row * kCols + qtr * 32 + ch * 4) = pk;
                  }
                }
              }
              if (hp8 && warp == 0 && lane == 0) a.hs[unit * nrb + t] = s8;
              fence_async_smem();
              __syncwarp();
              const int wrows = min(8, rows - row0);
              if (lane == 0 && wrows > 0) {
                const int esz_hp = hp16 ? 2 : hp8 ? 1 : 4;
                bulk_s2g(static_cast<unsigned char *>(a.hp) + (unit * R + kFp4Rows * t + row0) * kCols * esz_hp,
                         stw + row0 * kCols * esz_hp, (uint32_t)(wrows * kCols * esz_hp), pol_wr);
                bulk_commit();
              }
            }
            if (fp4_read) {
              const float g = nvfp4_tile_scale(tmax);
              if (warp == 0 && lane == 0) a.rg[unit * nrb + t] = g;
              if (live && fp4d) {  // two-axis copy: the blocks are formed on x' = x / k
                const float *kr = kvals + (row >> 4) * kCols + qtr * 32;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const float4 k4 = *reinterpret_cast<const float4 *>(kr + ((c + lane) & 7) * 4);
                  sv[c].x = k4.x > 0.f ? __fdiv_rn(sv[c].x, k4.x) : 0.f;
                  sv[c].y = k4.y > 0.f ? __fdiv_rn(sv[c].y, k4.y) : 0.f;
                  sv[c].z = k4.z > 0.f ? __fdiv_rn(sv[c].z, k4.z) : 0.f;
                  sv[c].w = k4.w > 0.f ? __fdiv_rn(sv[c].w, k4.w) : 0.f;
                }
              }
              if (live) {
                // this lane's 32 columns are blocks qtr*2 and qtr*2+1; chunk ch lies in block ch >> 2
                float bam0 = 0.f, bam1 = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const int ch = (c + lane) & 7;
                  const float mq = fmaxf(fmaxf(fabsf(sv[c].x), fabsf(sv[c].y)), fmaxf(fabsf(sv[c].z), fabsf(sv[c].w)));
                  if (ch < 4) bam0 = fmaxf(bam0, mq); else bam1 = fmaxf(bam1, mq);
                }
                float db0, db1;
                const uint32_t sc0 = fp4d ? nvfp4d_block_scale(bam0, &db0) : nvfp4_block_scale(bam0, g, &db0);
                const uint32_t sc1 = fp4d ? nvfp4d_block_scale(bam1, &db1) : nvfp4_block_scale(bam1, g, &db1);
                *reinterpret_cast<uint16_t *>(a.rs + (unit * R + rowg) * (kCols / 16) + qtr * 2) =
                    (uint16_t)(sc0 | (sc1 << 8));
                unsigned char *cd = a.rq + (unit * R + rowg) * (kCols / 2) + qtr * 16;
                const float rb0 = __frcp_rn(db0), rb1 = __frcp_rn(db1);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const int ch = (c + lane) & 7;
                  const uint32_t cw = nvfp4_code4(sv[c], ch < 4 ? db0 : db1, ch < 4 ? rb0 : rb1);
                  *reinterpret_cast<uint16_t *>(cd + ch * 2) = (uint16_t)cw;
                }
              }
            }
          }
          if (lane == 0) bulk_wait_read();  // a bulk store of this stage must have read it before release
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
    for (int s = 0; s < 8; ++s)
      if (armed[s] >= 0) mbar_wait(&full[s], (uint32_t)(armed[s] & 1), ws);
    for (int s = 0; s < kGBG; ++s)
      if (armed[8 + s] >= 0) mbar_wait(&gfull[s], (uint32_t)(armed[8 + s] & 1), ws);
  }
  if (threadIdx.x == 0) sched_finish(a.err);
}

}  // namespace

static bool g_lowprec(int hp_mode, int read_mode) { return hp_mode != RSSM_HP_F32 || read_mode != RSSM_READ_SAME; }

int g_smem_bytes(int R, int L, int tmax, int esz, int nstage, int hp_mode, int read_mode) {
  const GLayout l = g_layout(R, L, tmax, esz, g_chunked(hp_mode, read_mode, esz, L));
  return kBarBytesG + 2 * l.tab_bytes + kGBG * l.gb_bytes + nstage * l.stage_bytes;
}

int g_max_stages(int R, int L, int tmax, int esz, int hp_mode, int read_mode, int budget) {
  int n = 8;
  while (n > 2 && g_smem_bytes(R, L, tmax, esz, n, hp_mode, read_mode) > budget) --n;
  return n;
}

int g_extra_smem_bytes(int L, int esz, int hp_mode, int read_mode) {
  (void)L;
  (void)esz;
  (void)hp_mode;
  return read_mode == RSSM_READ_NVFP4D ? kCmBytes : 0;
}

int g_units(int Bt, int H, int tmax) {
  const int no = tmax <= 1 ? 1 : tmax <= 2 ? 2 : tmax <= 4 ? 4 : 8;
  const int hg = g_heads_per_unit(no);
  return Bt * ((H + hg - 1) / hg);
}

cudaError_t launch_gdn_replay(GArgs a, int esz, cudaStream_t stream) {
  const int no = a.tmax <= 1 ? 1 : a.tmax <= 2 ? 2 : a.tmax <= 4 ? 4 : 8;
  const size_t smem = g_smem_bytes(a.DV, a.L, a.tmax, esz, a.nstage, a.hp_mode, a.read_mode) +
                      g_extra_smem_bytes(a.L, esz, a.hp_mode, a.read_mode);
  void (*kern)(GArgs) = nullptr;
  const bool lp = g_lowprec(a.hp_mode, a.read_mode);
  // the low-precision instance with the chunked fold serves the fp32 checkpoint with an NVFP4 read copy, at
  // steps that may fold
  const bool lpc = lp && g_chunked(a.hp_mode, a.read_mode, esz, a.L) && !a.fold_free;
#define RSSM_PICK(TI, NOV, CFV)                                                                    \
  if (no == NOV)                                                                                   \
    kern = lp ? (CFV && lpc ? gdn_replay_kernel<TI, NOV, true, CFV> : gdn_replay_kernel<TI, NOV, true, false>) \
              : gdn_replay_kernel<TI, NOV, false, CFV>;
  if (esz == 2) {
    RSSM_PICK(__nv_bfloat16, 1, true) RSSM_PICK(__nv_bfloat16, 2, true) RSSM_PICK(__nv_bfloat16, 4, true)
    RSSM_PICK(__nv_bfloat16, 8, true)
    if (no == 1 && !lp && a.fold_free) kern = gdn_replay_kernel<__nv_bfloat16, 1, false, false>;
  } else {
    RSSM_PICK(float, 1, false) RSSM_PICK(float, 2, false) RSSM_PICK(float, 4, false) RSSM_PICK(float, 8, false)
  }
#undef RSSM_PICK
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<a.grid, kGdnThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rssm
