/*
 * rssm.h -- C ABI of the ReplaySSM decode library (B200, sm_100a).
 *
 * ReplaySSM keeps the recurrent state of a state-space layer as a checkpoint
 * plus a buffer of the inputs of the last <= L tokens.  A decode step appends
 * its inputs and computes its output from checkpoint and buffer without
 * writing state back; only a full buffer is folded into a new checkpoint.
 * Sources (news pages about the paper "ReplaySSM: Cache SSM Inputs, Not
 * State"):
 *   [HMD] "Hybrid-model decoding has a new bottleneck: stop writing the SSM
 *         state every step, and speculative throughput reaches 2.10x"
 *         (ai4snews): Synopsis; Interpretation paragraphs 2-4; Perspective.
 *   [NVD] "NVIDIA and Dao AI Lab speed up hybrid-model decoding"
 *         (aimodeltracker): third paragraph.
 *   [SSD] "SSM decoding stops writing state every step: caching recent inputs
 *         halves state traffic and matches vLLM speculation" (ai4snews):
 *         Synopsis; Interpretation paragraphs 2-3; Perspective.
 * plus the published Mamba-2 and gated-delta-rule recurrences:
 *   Mamba-2, per head h of group g(h), S in R^{P x N}:
 *       S_t = exp(dt_t A_h) S_{t-1} + dt_t x_t B_t^T,  y_t = S_t C_t + D_h x_t
 *   Gated DeltaNet, S in R^{d_v x d_k}:
 *       S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *       y_t = q_scale S_t q_t
 *
 * Conventions for every call below
 *   - Pointers named "device" point to device memory of the current device;
 *     the library never allocates, frees or copies device memory on its own
 *     behalf except inside the caller's arena.  Host pointers are named so.
 *   - Calls are asynchronous on the given stream (NULL = legacy default
 *     stream) unless stated; they return after the launch.
 *   - Host-checkable errors (null or misaligned pointers, unsupported shapes,
 *     out-of-range arguments) return a status without launching anything.
 *   - Errors detected on the device (a call that the per-sequence state
 *     forbids, e.g. a commit without a pending verify) never trap: the
 *     offending sequence is left untouched, its outputs are not written, and
 *     a sticky error word records the lowest failing sequence index and its
 *     code; read it with rssm_get_error.
 *   - Calls on one context must be ordered on one stream (or ordered by the
 *     caller with events); the library flips an internal parity bit on every
 *     call that changes the bookkeeping.
 *   - Token inputs are row-major with the leading dimensions named, and must
 *     start on 16-byte boundaries; rows of length P, N, d_k or d_v in the
 *     input dtype must be multiples of 16 bytes.
 */
#ifndef RSSM_H
#define RSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *rssm_stream; /* a cudaStream_t */

typedef enum {
  RSSM_OK = 0,
  RSSM_ERR_ARG = 1,             /* null / misaligned pointer, bad enum or count */
  RSSM_ERR_SHAPE = 2,           /* a dimension outside the supported set */
  RSSM_ERR_UNSUPPORTED = 3,     /* call not valid for this context's kind or mode */
  RSSM_ERR_ARENA_TOO_SMALL = 4, /* arena smaller than rssm_arena_bytes */
  RSSM_ERR_CUDA = 5,            /* a CUDA runtime call failed; see rssm_last_cuda_error */
  RSSM_ERR_DEVICE = 6           /* rssm_get_error found a recorded device-side error */
} rssm_status;

/* device-side error codes reported by rssm_get_error */
enum {
  RSSM_DEV_OK = 0,
  RSSM_DEV_PENDING = 1,     /* step / verify / flush on a sequence with a verify pending */
  RSSM_DEV_NO_VERIFY = 2,   /* commit on a sequence without a pending verify */
  RSSM_DEV_ACCEPTED = 3,    /* accepted length outside 0..pending */
  RSSM_DEV_TIMEOUT = 4      /* a bounded wait on an asynchronous copy gave up */
};

typedef enum { RSSM_MAMBA2 = 0, RSSM_GDN = 1 } rssm_kind;
typedef enum { RSSM_F32 = 0, RSSM_BF16 = 1 } rssm_dtype;
/* precision of the recurrence checkpoint ([HMD] Interpretation 4th paragraph, Perspective 2nd;
 * FP8: [SSD] Interpretation 3rd paragraph): fp32; fp16 with stochastic rounding; or E4M3 (FP8)
 * times one fp32 scale amax/448 per 64-row tile of a head's state, rounded stochastically with
 * the same random words (GDN only) */
typedef enum { RSSM_HP_F32 = 0, RSSM_HP_F16_SR = 1, RSSM_HP_F8_SR = 2 } rssm_hp;
/* copy read for outputs: the checkpoint itself, a separate NVFP4 copy, (contrast only) one
 * NVFP4 copy that is also the checkpoint the recurrence continues from, or a separate NVFP4
 * copy with scales along both axes ([HMD] Interpretation 4th paragraph: separate scales along
 * the state and channel dimensions): an E4M3 scale per column for every 16 rows of a tile,
 * times the E4M3 block scales along each row (GDN only) */
typedef enum { RSSM_READ_SAME = 0, RSSM_READ_NVFP4 = 1, RSSM_READ_SHARED_NVFP4 = 2, RSSM_READ_NVFP4D = 3 } rssm_read;

typedef struct {
  int kind;        /* rssm_kind */
  int batch;       /* sequences, >= 1 */
  int nheads;      /* H */
  int headdim;     /* Mamba-2: P; GDN: d_v.  Rows of one head's state, 8..64 (Mamba-2) or 8..128 (GDN), multiple of 8 */
  int dstate;      /* Mamba-2: N; GDN: d_k.  Contiguous axis of the state; must be 128 */
  int ngroups;     /* Mamba-2: G, H % G == 0, head h reads group h / (H/G).  GDN: 1 */
  int window;      /* L, 1..32: tokens buffered before the checkpoint is folded */
  int max_draft;   /* T_max, 0..min(L, 8): largest speculative draft count for rssm_verify */
  int in_dtype;    /* rssm_dtype of x, B, C, dt (Mamba-2) or q, k, v (GDN); alpha, beta are fp32 */
  int hp;          /* rssm_hp */
  int read;        /* rssm_read */
  unsigned long long seed; /* key of the stochastic-rounding generator (Philox4x32-10) */
  float q_scale;   /* GDN output scale (y = q_scale * S q) */
  const float *A;  /* Mamba-2: device [H], A_h < 0; must stay valid while the context is used */
  const float *D;  /* Mamba-2: device [H] */
  float skip_tau;  /* GDN decay-aware read skipping ([SSD] Perspective 1st paragraph); 0 = off.  After
                    * each step, verify or flush, a head is flagged iff the fp32 product of alpha over the
                    * committed records of its window (in record order) is below skip_tau; the next call
                    * then neither reads that head's checkpoint nor its read copy (the term counts as
                    * zero, at most skip_tau * |S0| * q_scale * |q| in norm), and a fold writes the new
                    * checkpoint from the buffer alone.  A fold that empties the window clears the flag.
                    * Must be finite and >= 0; Mamba-2 requires 0. */
} rssm_config;

typedef struct rssm_ctx rssm_ctx;

/* Token inputs of rssm_verify, leading dims [batch][T]; unused members may be NULL. */
typedef struct {
  const void *x, *B, *C, *dt;      /* Mamba-2: x [Bt][T][H][P], B, C [Bt][T][G][N], dt [Bt][T][H] */
  const void *q, *k, *v;           /* GDN: q, k [Bt][T][H][d_k], v [Bt][T][H][d_v] */
  const float *alpha, *beta;       /* GDN: [Bt][T][H] */
} rssm_tokens;

/* ---------------------------------------------------------------- set-up (host only) */

/* Bytes of device memory a context needs (checkpoint, read copy, input ring, bookkeeping). */
rssm_status rssm_arena_bytes(const rssm_config *cfg, size_t *bytes);

/* Create a context over a caller-owned device arena (256-byte aligned, >= rssm_arena_bytes).
 * Only the small host handle is allocated (malloc).  The arena contents are undefined
 * until rssm_load_checkpoint: until its first success, every other call on the context
 * (decode, commit, flush, export, rssm_get_error) returns RSSM_ERR_UNSUPPORTED. */
rssm_status rssm_create(const rssm_config *cfg, void *arena, size_t arena_bytes, rssm_ctx **out);

/* Free the host handle.  The arena stays the caller's. */
rssm_status rssm_destroy(rssm_ctx *ctx);

/* Message of the last CUDA error seen by the library on this thread (static string). */
const char *rssm_last_cuda_error(void);

/* Load a checkpoint: S device fp32 [Bt][H][rows][cols] (rows = P or d_v, cols = N or d_k).
 * Writes it in the checkpoint format (fp32, or fp16 with stochastic rounding at epoch 0),
 * builds the NVFP4 read copy if the mode has one, empties every buffer (count = epoch =
 * pending = 0) and clears the error word.  [SSD] Synopsis: the checkpoint is the state
 * the buffered inputs are replayed against. */
rssm_status rssm_load_checkpoint(rssm_ctx *ctx, const float *S, rssm_stream stream);

/* ---------------------------------------------------------------- decode (device work) */

/* One Mamba-2 decode token per sequence.  [SSD] Interpretation 2nd paragraph: append the
 * token's inputs and compute y from checkpoint and buffer; [NVD] 3rd paragraph: only a
 * full buffer writes a new checkpoint.  Per sequence: if count == L (possible only after a
 * commit) the buffer is folded first; the record (x, B, dt) is stored in slot count;
 * count += 1; if count == L the buffer is folded now and y comes from the new state,
 * otherwise
 *   y = exp(A sum_i dt_i) S0 C + sum_i exp(A sum_{j>i} dt_j) dt_i (B_i . C) x_i + D x
 * over the buffered tokens i (the current one last).
 *   x  device [Bt][H][P], B, C device [Bt][G][N], dt device [Bt][H] (post-activation),
 *      all in cfg.in_dtype;  y device fp32 [Bt][H][P], written for every sequence that
 *      has no verify pending. */
rssm_status rssm_mamba2_step(rssm_ctx *ctx, const void *x, const void *B, const void *C, const void *dt,
                             float *y, rssm_stream stream);

/* One Gated DeltaNet decode token per sequence.  Same bookkeeping as rssm_mamba2_step.
 * The output walks q back through the buffered factors alpha_i (I - beta_i k_i k_i^T)
 * (newest first), collecting sum_i beta_i c_i v_i with c_i = k_i . u_i, and then reads the
 * checkpoint with one matrix-vector product: y = q_scale (S0 u_0 + sum_i beta_i c_i v_i).
 *   q, k device [Bt][H][d_k], v device [Bt][H][d_v] (cfg.in_dtype);
 *   alpha, beta device fp32 [Bt][H];  y device fp32 [Bt][H][d_v]. */
rssm_status rssm_gdn_step(rssm_ctx *ctx, const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, float *y, rssm_stream stream);

/* Speculative verification of T draft tokens (1 <= T <= cfg.max_draft).  [HMD] Interpretation
 * 3rd paragraph, [SSD] Interpretation 3rd paragraph: outputs only, no per-draft state.
 * Per sequence: if count + T > L the committed records are folded first; the drafts go to
 * slots count..count+T-1 without moving count; y for every draft is computed from the
 * checkpoint and the buffer; pending = T.
 *   tok: inputs with leading dims [Bt][T];  y device fp32 [Bt][T][H][rows]. */
rssm_status rssm_verify(rssm_ctx *ctx, int T, const rssm_tokens *tok, float *y, rssm_stream stream);

/* Commit the accepted prefix of the pending drafts: count += accepted[b], pending = 0.
 * A buffer-pointer move; nothing else is written ([HMD] Interpretation 3rd paragraph).
 *   accepted device int32 [Bt], each in 0..pending[b]. */
rssm_status rssm_commit(rssm_ctx *ctx, const int *accepted, rssm_stream stream);

/* Fold the committed records of the selected sequences into the checkpoint (count = 0,
 * epoch += 1 where count > 0).  mask device uint8 [Bt] (nonzero = selected) or NULL = all. */
rssm_status rssm_flush(rssm_ctx *ctx, const unsigned char *mask, rssm_stream stream);

/* ---------------------------------------------------------------- inspection */

/* Bytes of the logical ring view written by rssm_export (may be 0 if ring_out is not wanted). */
rssm_status rssm_ring_bytes(const rssm_config *cfg, size_t *bytes);

/* Copy the state out (device destinations, any may be NULL):
 *   S_out fp32 [Bt][H][rows][cols]: the stored checkpoint, widened to fp32;
 *   ring_out: the current window's slots 0..L-1 in the input dtype, concatenated as
 *     Mamba-2: x [Bt][H][L][P], B [Bt][G][L][N], dt [Bt][H][L] (fp32);
 *     GDN: k [Bt][H][L][d_k], v [Bt][H][L][d_v], alpha [Bt][H][L], beta [Bt][H][L] (fp32);
 *   meta_out int32 [Bt][4]: count, epoch, pending, window base slot. */
rssm_status rssm_export(rssm_ctx *ctx, float *S_out, void *ring_out, int *meta_out, rssm_stream stream);

/* Copy the NVFP4 read copy out (device destinations): codes uint8 [Bt][H][rows][cols/2]
 * (element 2j in the low nibble), scales uint8 [Bt][H][rows][cols/16] (E4M3 of each
 * 16-element block), g fp32 [Bt][H][ceil(rows/64)] (one scale per 64-row tile).
 * RSSM_ERR_UNSUPPORTED if the context has no read copy. */
rssm_status rssm_export_read_copy(rssm_ctx *ctx, unsigned char *codes, unsigned char *scales, float *g,
                                  rssm_stream stream);

/* Copy the column-group scales of a two-axis read copy (RSSM_READ_NVFP4D) out: colscales uint8
 * [Bt][H][ceil(rows/16)][128] (device), the E4M3 scale of each column for each group of 16 rows;
 * rssm_export_read_copy gives its codes, row-block scales and tile scales (the row-block scale of
 * this copy is d_b = E4M3 * 2^-8, in units of the column-group step E4M3 * g).
 * RSSM_ERR_UNSUPPORTED for any other read mode. */
rssm_status rssm_export_column_scales(rssm_ctx *ctx, unsigned char *colscales, rssm_stream stream);

/* Copy the decay-aware skip flags out: flags uint8 [Bt][H] (device), 1 = the next call skips
 * that head's checkpoint read.  RSSM_ERR_UNSUPPORTED if the context has skip_tau == 0. */
rssm_status rssm_export_skip(rssm_ctx *ctx, unsigned char *flags, rssm_stream stream);

/* Synchronise the stream and read the sticky device error word: *code (RSSM_DEV_*) and
 * *seq (lowest failing sequence, -1 if none).  Returns RSSM_ERR_DEVICE if one is set. */
rssm_status rssm_get_error(rssm_ctx *ctx, int *code, int *seq, rssm_stream stream);

/* ---------------------------------------------------------------- comparison kernels
 * In-house conventional kernels that read and write the full state every token, the
 * scheme the pages measure against ([HMD] Interpretation 2nd and 3rd paragraphs).
 * They use only cfg's shape fields (kind, batch, nheads, headdim, dstate, ngroups,
 * in_dtype, q_scale, A, D). */

/* Conventional step: S device fp32 [Bt][H][rows][cols], read and rewritten in place. */
rssm_status rssm_conv_mamba2_step(const rssm_config *cfg, float *S, const void *x, const void *B, const void *C,
                                  const void *dt, float *y, rssm_stream stream);
rssm_status rssm_conv_gdn_step(const rssm_config *cfg, float *S, const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta, float *y, rssm_stream stream);

/* Snapshot-per-draft speculation: snaps device fp32 [Bt][T_max+1][H][rows][cols], the live
 * state of sequence b in slot cur[b] (device int32 [Bt]).  Verify reads the live slot once
 * and writes the state after draft j to slot (cur[b] + j + 1) % (T_max + 1); commit moves
 * cur[b] to the accepted draft's slot.  T_max = cfg.max_draft. */
rssm_status rssm_snap_verify(const rssm_config *cfg, float *snaps, const int *cur, int T, const rssm_tokens *tok,
                             float *y, rssm_stream stream);
rssm_status rssm_snap_commit(const rssm_config *cfg, int *cur, const int *accepted, rssm_stream stream);

/* ---------------------------------------------------------------- scheduler self-test */

/* Run the unit scheduler of the replay kernels on its own: `blocks` blocks draw `units` work
 * units from a counter with one atomic per unit, and the last block to finish re-arms the
 * counter (the mechanism the replay kernels use on the counter in the context's arena).  The
 * pages have no counterpart: this is a check of this library's own scheduling.
 *
 * It allocates nothing and needs no caller device memory, for callers that cannot allocate
 * on the device (for instance a process that only holds a driver context, or code running
 * where device allocation is forbidden): the counter, per-unit claim marks and per-block
 * tallies live in one file-scope device array of the library, of fixed size (about 260 KiB,
 * for at most 65536 units and 1024 blocks), which every device that loads the library holds
 * until the process exits.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with the device current); make that first call before any stream
 * capture.  Every call clears the array before use, and all calls share it: calls that
 * overlap on the GPU race, so order them on one stream.
 *   units 1 .. 65536, blocks 1 .. 1024 (RSSM_ERR_ARG beyond these limits, before any device work);
 *   per_block host int [blocks]: units each block drew (they sum to `units`);
 *   bad_units host int [1]: units not drawn exactly once, plus one if the last block did not
 *     re-arm the counter (0 when correct).
 * Synchronises `stream`.  RSSM_ERR_ARG on a count out of range or a null pointer. */
rssm_status rssm_sched_probe(int units, int blocks, int *per_block, int *bad_units, rssm_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* RSSM_H */
