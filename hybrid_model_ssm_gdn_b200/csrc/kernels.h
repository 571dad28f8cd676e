// kernels.h -- launch interfaces between the host API (api.cu) and the kernels.
#pragma once

#include "common.cuh"

namespace rssm {

enum { OP_STEP = 0, OP_VERIFY = 1, OP_FLUSH = 2 };

// Mamba-2 replay kernel (step / verify / flush).  Pointers are device pointers.
struct M2Args {
  int Bt, H, P, G, L;
  int T;          // tokens per sequence in this call (1 step, T verify, 0 flush)
  int tmax;       // sizes the per-stage record area: L + max(tmax, 1) records
  int op;
  int units;      // Bt * H
  int fold_free;  // the host knows that no unit of this launch folds (the instance without the chunked fold)
  int grid, nstage, stage_base;
  const int4 *meta_in;
  int4 *meta_out;
  int *err;
  float *hp;                      // fp32 [Bt][H][P][128]
  void *ring_x, *ring_B;          // input dtype [Bt][H][2L][P], [Bt][G][2L][128]
  float *ring_dt;                 // [Bt][H][dt_stride(L)]
  const void *x, *Bin, *C, *dt;   // [Bt][T][H][P], [Bt][T][G][128] x2, [Bt][T][H]
  const unsigned char *mask;      // flush only, may be null
  const float *A, *D;
  float *y;                       // [Bt][T][H][P]
  unsigned char *skip;            // decay-aware skip flags [Bt][H], or null when skipping is off
  float skip_ln_tau;              // flag threshold on A_h times the sum of dt over the committed records
  long long wait_cycles;          // bound of every wait on an asynchronous copy or another warp
  unsigned int suspend_ns;        // suspend-time hint of each try_wait (0: the hardware's default)
  int withhold;                   // test hook: no block fills its tile with this index (-1: off)
};
int m2_smem_bytes(int P, int L, int tmax, int esz, int nstage);
int m2_max_stages(int P, int L, int tmax, int esz, int smem_budget);
int m2_units(int Bt, int H, int G);  // work units: (sequence, group chunk of <= 16 heads)
cudaError_t launch_m2_replay(M2Args a, int esz, cudaStream_t stream);

// Gated DeltaNet replay kernel (step / verify / flush) with the precision modes.
struct GArgs {
  int Bt, H, DV, L;
  int T, tmax, op, units, grid, nstage, stage_base;
  int fold_free;  // the host knows that no unit of this launch folds (the instance without the chunked fold)
  int hp_mode, read_mode;         // rssm_hp, rssm_read
  unsigned long long seed;
  float q_scale;
  const int4 *meta_in;
  int4 *meta_out;
  int *err;
  void *hp;                       // fp32, fp16 or E4M3 [Bt][H][DV][128]
  float *hs;                      // E4M3 checkpoint tile scales [Bt][H][ceil(DV/64)]
  unsigned char *rq, *rs;         // NVFP4 codes [Bt][H][DV][64], scales [Bt][H][DV][8]
  float *rg;                      // tile scales [Bt][H][ceil(DV/64)]
  unsigned char *rc;              // two-axis copy: column-group scales [Bt][H][ceil(DV/16)][128]
  unsigned char *skip;            // decay-aware skip flags [Bt][H], or null when skipping is off
  float skip_tau;                 // flag threshold on the product of alpha over the committed records
  void *ring_k, *ring_v;          // input dtype [Bt][H][2L][128], [Bt][H][2L][DV]
  float *ring_a, *ring_b;         // alpha, beta [Bt][H][dt_stride(L)]
  const void *q, *k, *v;          // [Bt][T][H][128], [Bt][T][H][128], [Bt][T][H][DV]
  const float *alpha, *beta;      // [Bt][T][H]
  const unsigned char *mask;
  float *y;                       // [Bt][T][H][DV]
  long long wait_cycles;          // bound of every wait on an asynchronous copy or another warp
  unsigned int suspend_ns;        // suspend-time hint of each try_wait (0: the hardware's default)
  int withhold;                   // test hook: no block fills its tile with this index (-1: off)
};
int g_smem_bytes(int R, int L, int tmax, int esz, int nstage, int hp_mode, int read_mode);
// fold scratch behind the stages: the two-axis read copy's column maxima, or the chunked fold's Z / W
int g_extra_smem_bytes(int L, int esz, int hp_mode, int read_mode);
int g_max_stages(int R, int L, int tmax, int esz, int hp_mode, int read_mode, int budget);
int g_units(int Bt, int H, int tmax);  // work units: (sequence, chunk of heads)
cudaError_t launch_gdn_replay(GArgs a, int esz, cudaStream_t stream);

// small kernels (bookkeeping, load, export)
cudaError_t launch_meta_reset(int4 *meta, int Bt, int *err, cudaStream_t stream);
cudaError_t launch_commit(const int4 *meta_in, int4 *meta_out, const int *accepted, int Bt, int *err,
                          cudaStream_t stream);
cudaError_t launch_export_meta(const int4 *meta, int *out, int Bt, int L, cudaStream_t stream);
cudaError_t launch_gather_window(const unsigned char *in, unsigned char *out, const int4 *meta, int Bt, int X,
                                 size_t in_group_bytes, int slot_bytes, int L, cudaStream_t stream);
cudaError_t launch_store_state(const float *S, void *hp, float *hs, int hp_mode, unsigned char *rq, unsigned char *rs,
                               float *rg, unsigned char *rc, int read_mode, int units, int rows, unsigned long long seed,
                               int H, cudaStream_t stream);
cudaError_t launch_widen_state(const void *hp, const float *hs, int hp_mode, const unsigned char *rq,
                               const unsigned char *rs, const float *rg, int read_mode, float *out, int units, int rows,
                               cudaStream_t stream);

// comparison kernels (conventional step, snapshot-per-draft)
struct ConvArgs {
  int kind, Bt, H, R, G, T, tmax;
  float q_scale;
  float *S;                      // conventional: [Bt][H][R][128]; snapshot: [Bt][tmax+1][H][R][128]
  const int *cur;                // snapshot: live slot per sequence (null for conventional)
  const void *x, *Bin, *C, *dt;  // Mamba-2 inputs [Bt][T][...]
  const void *q, *k, *v;         // GDN inputs [Bt][T][...]
  const float *alpha, *beta;
  const float *A, *D;
  float *y;                      // [Bt][T][H][R]
};
cudaError_t launch_conv(ConvArgs a, int esz, cudaStream_t stream);
cudaError_t launch_snap_commit(int *cur, const int *accepted, int Bt, int nslots, cudaStream_t stream);

}  // namespace rssm
