// api.cu -- host side of the C ABI declared in include/rssm.h.
//
// Validates arguments, carves the caller's arena, keeps the bookkeeping parity bit and
// launches the kernels on the caller's stream.  Nothing here allocates device memory.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kernels.h"
#include "sched.h"

using namespace rssm;

struct rssm_ctx {
  rssm_config cfg;
  ArenaLayout lay;
  unsigned char *arena;
  int parity;    // meta[parity] is current
  int num_sms;
  int smem_optin;
  int nstage_override;
  int loaded;    // set by the first successful rssm_load_checkpoint
  float skip_ln_tau;       // Mamba-2 decay-aware skipping: ln(skip_tau) in fp32
  long long wait_cycles;   // bound of the kernels' waits (RSSM_WAIT_CYCLES, default ~1 s)
  unsigned int suspend_ns; // suspend-time hint of the kernels' barrier polls (RSSM_SUSPEND_NS)
  int withhold;            // test hook RSSM_WITHHOLD_TILE (-1: off)
  // every sequence's record count in the window when the host knows it (only steps since the checkpoint was
  // loaded or fully flushed), else -1.  It picks the kernel instance of a step; both fold correctly.
  int pos;
};

namespace {

thread_local char g_last_cuda_error[256] = "no error";

rssm_status cuda_fail(cudaError_t e) {
  snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return RSSM_ERR_CUDA;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int esize(const rssm_config &c) { return c.in_dtype == RSSM_BF16 ? 2 : 4; }

rssm_status validate(const rssm_config *c) {
  if (!c) return RSSM_ERR_ARG;
  if (c->kind != RSSM_MAMBA2 && c->kind != RSSM_GDN) return RSSM_ERR_ARG;
  if (c->in_dtype != RSSM_F32 && c->in_dtype != RSSM_BF16) return RSSM_ERR_ARG;
  if (c->hp != RSSM_HP_F32 && c->hp != RSSM_HP_F16_SR && c->hp != RSSM_HP_F8_SR) return RSSM_ERR_ARG;
  if (c->read < RSSM_READ_SAME || c->read > RSSM_READ_NVFP4D) return RSSM_ERR_ARG;
  if (!(c->skip_tau >= 0.f) || c->skip_tau > 3.0e38f) return RSSM_ERR_ARG;  // NaN, negative or infinite
  if (c->batch < 1 || c->nheads < 1) return RSSM_ERR_SHAPE;
  if ((long long)c->batch * c->nheads > (1LL << 26)) return RSSM_ERR_SHAPE;
  if (c->dstate != kCols) return RSSM_ERR_SHAPE;
  if (c->headdim < 8 || c->headdim % 8 != 0) return RSSM_ERR_SHAPE;
  if (c->window < 1 || c->window > kMaxWindow) return RSSM_ERR_SHAPE;
  const int tcap = c->window < kMaxDraft ? c->window : kMaxDraft;
  if (c->max_draft < 0 || c->max_draft > tcap) return RSSM_ERR_SHAPE;
  if (c->kind == RSSM_MAMBA2) {
    if (c->headdim > 64) return RSSM_ERR_SHAPE;
    if (c->ngroups < 1 || c->nheads % c->ngroups != 0) return RSSM_ERR_SHAPE;
    if (!c->A || !c->D) return RSSM_ERR_ARG;
    if (c->hp != RSSM_HP_F32 || c->read != RSSM_READ_SAME) return RSSM_ERR_UNSUPPORTED;
  } else {
    if (c->headdim > 128) return RSSM_ERR_SHAPE;
    if (c->ngroups != 1) return RSSM_ERR_SHAPE;
  }
  return RSSM_OK;
}

// a step the host knows to fold nowhere: every sequence's count is known and stays below the window
bool known_fold_free(const rssm_ctx *x, int op) { return op == OP_STEP && x->pos >= 0 && x->pos + 1 < x->cfg.window; }

// the record count after a successful call (rssm_ctx::pos)
void advance_pos(rssm_ctx *x, int op, const unsigned char *mask) {
  if (op == OP_STEP && x->pos >= 0) x->pos = x->pos + 1 == x->cfg.window ? 0 : x->pos + 1;
  else if (op == OP_FLUSH && mask == nullptr) x->pos = 0;
  else x->pos = -1;
}

const int4 *meta_cur(rssm_ctx *x) { return reinterpret_cast<const int4 *>(x->arena + x->lay.meta) + x->parity * x->cfg.batch; }
int4 *meta_next(rssm_ctx *x) { return reinterpret_cast<int4 *>(x->arena + x->lay.meta) + (1 - x->parity) * x->cfg.batch; }
int *err_word(rssm_ctx *x) { return reinterpret_cast<int *>(x->arena + x->lay.err); }

rssm_status run_m2(rssm_ctx *x, int op, int T, const void *xin, const void *B, const void *C, const void *dt,
                   const unsigned char *mask, float *y, cudaStream_t stream) {
  if (!x->loaded) return RSSM_ERR_UNSUPPORTED;
  const rssm_config &c = x->cfg;
  M2Args a{};
  a.Bt = c.batch; a.H = c.nheads; a.P = c.headdim; a.G = c.ngroups; a.L = c.window;
  a.T = T; a.tmax = op == OP_VERIFY ? T : 1; a.op = op;
  a.units = m2_units(c.batch, c.nheads, c.ngroups);
  a.fold_free = known_fold_free(x, op);
  a.grid = a.units < x->num_sms ? a.units : x->num_sms;
  const int esz = esize(c);
  a.nstage = x->nstage_override > 0 ? x->nstage_override : m2_max_stages(a.P, a.L, a.tmax, esz, x->smem_optin - 1024);
  if (a.nstage < 2 || a.nstage > 8 || m2_smem_bytes(a.P, a.L, a.tmax, esz, a.nstage) > x->smem_optin) return RSSM_ERR_SHAPE;
  a.meta_in = meta_cur(x); a.meta_out = meta_next(x); a.err = err_word(x);
  a.hp = reinterpret_cast<float *>(x->arena + x->lay.hp);
  a.ring_x = x->arena + x->lay.ring_a; a.ring_B = x->arena + x->lay.ring_b;
  a.ring_dt = reinterpret_cast<float *>(x->arena + x->lay.ring_c);
  a.x = xin; a.Bin = B; a.C = C; a.dt = dt; a.mask = mask; a.A = c.A; a.D = c.D; a.y = y;
  a.skip = c.skip_tau > 0.f ? x->arena + x->lay.skip : nullptr;
  a.skip_ln_tau = x->skip_ln_tau;
  a.wait_cycles = x->wait_cycles; a.suspend_ns = x->suspend_ns; a.withhold = x->withhold;
  x->withhold = -1;  // the test hook fires on one launch only
  cudaError_t e = launch_m2_replay(a, esz, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->parity ^= 1;
  advance_pos(x, op, mask);
  return RSSM_OK;
}

rssm_status run_gdn(rssm_ctx *x, int op, int T, const void *q, const void *k, const void *v, const float *alpha,
                    const float *beta, const unsigned char *mask, float *y, cudaStream_t stream) {
  if (!x->loaded) return RSSM_ERR_UNSUPPORTED;
  const rssm_config &c = x->cfg;
  GArgs a{};
  a.Bt = c.batch; a.H = c.nheads; a.DV = c.headdim; a.L = c.window;
  a.T = T; a.tmax = op == OP_VERIFY ? T : 1; a.op = op;
  a.units = g_units(c.batch, c.nheads, a.tmax);
  a.fold_free = known_fold_free(x, op);
  a.grid = a.units < x->num_sms ? a.units : x->num_sms;
  a.hp_mode = c.hp; a.read_mode = c.read; a.seed = c.seed; a.q_scale = c.q_scale;
  const int esz = esize(c);
  const int extra = g_extra_smem_bytes(a.L, esz, c.hp, c.read);
  a.nstage = x->nstage_override > 0 ? x->nstage_override
                                    : g_max_stages(a.DV, a.L, a.tmax, esz, c.hp, c.read, x->smem_optin - 1024 - extra);
  if (a.nstage < 2 || a.nstage > 8 ||
      g_smem_bytes(a.DV, a.L, a.tmax, esz, a.nstage, c.hp, c.read) + extra > x->smem_optin)
    return RSSM_ERR_SHAPE;
  a.meta_in = meta_cur(x); a.meta_out = meta_next(x); a.err = err_word(x);
  a.hp = x->arena + x->lay.hp;
  a.hs = reinterpret_cast<float *>(x->arena + x->lay.hs);
  a.rq = x->arena + x->lay.rq; a.rs = x->arena + x->lay.rs; a.rg = reinterpret_cast<float *>(x->arena + x->lay.rg);
  a.rc = x->arena + x->lay.rc;
  a.ring_k = x->arena + x->lay.ring_a; a.ring_v = x->arena + x->lay.ring_b;
  a.ring_a = reinterpret_cast<float *>(x->arena + x->lay.ring_c);
  a.ring_b = reinterpret_cast<float *>(x->arena + x->lay.ring_d);
  a.skip = c.skip_tau > 0.f ? x->arena + x->lay.skip : nullptr;
  a.skip_tau = c.skip_tau;
  a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.mask = mask; a.y = y;
  a.wait_cycles = x->wait_cycles; a.suspend_ns = x->suspend_ns; a.withhold = x->withhold;
  x->withhold = -1;  // the test hook fires on one launch only
  cudaError_t e = launch_gdn_replay(a, esz, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->parity ^= 1;
  advance_pos(x, op, mask);
  return RSSM_OK;
}

}  // namespace

extern "C" {

const char *rssm_last_cuda_error(void) { return g_last_cuda_error; }

rssm_status rssm_arena_bytes(const rssm_config *cfg, size_t *bytes) {
  rssm_status s = validate(cfg);
  if (s != RSSM_OK) return s;
  if (!bytes) return RSSM_ERR_ARG;
  *bytes = make_layout(*cfg).total;
  return RSSM_OK;
}

rssm_status rssm_ring_bytes(const rssm_config *cfg, size_t *bytes) {
  rssm_status s = validate(cfg);
  if (s != RSSM_OK) return s;
  if (!bytes) return RSSM_ERR_ARG;
  const size_t Bt = cfg->batch, H = cfg->nheads, L = cfg->window, R = cfg->headdim, esz = esize(*cfg);
  if (cfg->kind == RSSM_MAMBA2)
    *bytes = Bt * H * L * R * esz + Bt * cfg->ngroups * L * kCols * esz + Bt * H * L * 4;
  else
    *bytes = Bt * H * L * kCols * esz + Bt * H * L * R * esz + 2 * Bt * H * L * 4;
  return RSSM_OK;
}

rssm_status rssm_create(const rssm_config *cfg, void *arena, size_t arena_bytes, rssm_ctx **out) {
  rssm_status s = validate(cfg);
  if (s != RSSM_OK) return s;
  if (!arena || !out || ((uintptr_t)arena & 255u)) return RSSM_ERR_ARG;
  const ArenaLayout lay = make_layout(*cfg);
  if (arena_bytes < lay.total) return RSSM_ERR_ARENA_TOO_SMALL;
  int dev = 0, sms = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  rssm_ctx *x = static_cast<rssm_ctx *>(calloc(1, sizeof(rssm_ctx)));
  if (!x) return RSSM_ERR_ARG;
  x->cfg = *cfg;
  x->lay = lay;
  x->arena = static_cast<unsigned char *>(arena);
  x->pos = -1;
  x->parity = 0;
  x->num_sms = sms;
  x->smem_optin = optin;
  const char *ns = getenv("RSSM_NSTAGE");
  x->nstage_override = ns ? atoi(ns) : 0;
  // the rule is A_h * sum(dt) < ln(tau) in fp32; ln is taken in double by the C library and rounded once
  x->skip_ln_tau = cfg->skip_tau > 0.f ? (float)log((double)cfg->skip_tau) : 0.f;
  x->wait_cycles = kWaitCycles;
  const char *wc = getenv("RSSM_WAIT_CYCLES");
  if (wc) {
    const long long v = atoll(wc);
    x->wait_cycles = v < 100000LL ? 100000LL : v > kWaitCycles ? kWaitCycles : v;
  }
  const char *sn = getenv("RSSM_SUSPEND_NS");
  x->suspend_ns = sn ? (unsigned)atoi(sn) : kSuspendNs;
  // test hook for the timeout path: honoured only together with a shortened wait bound
  const char *wh = getenv("RSSM_WITHHOLD_TILE");
  x->withhold = (wh && wc) ? atoi(wh) : -1;
  *out = x;
  return RSSM_OK;
}

rssm_status rssm_destroy(rssm_ctx *ctx) {
  if (!ctx) return RSSM_ERR_ARG;
  free(ctx);
  return RSSM_OK;
}

rssm_status rssm_load_checkpoint(rssm_ctx *x, const float *S, rssm_stream stream) {
  if (!x || !S || !aligned16(S)) return RSSM_ERR_ARG;
  const rssm_config &c = x->cfg;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t units = (size_t)c.batch * c.nheads;
  cudaError_t e;
  if (c.hp == RSSM_HP_F32 && c.read == RSSM_READ_SAME)
    e = cudaMemcpyAsync(x->arena + x->lay.hp, S, units * c.headdim * kCols * 4, cudaMemcpyDeviceToDevice, st);
  else
    e = launch_store_state(S, x->arena + x->lay.hp, reinterpret_cast<float *>(x->arena + x->lay.hs), c.hp,
                           x->arena + x->lay.rq, x->arena + x->lay.rs,
                           reinterpret_cast<float *>(x->arena + x->lay.rg), x->arena + x->lay.rc, c.read, (int)units,
                           c.headdim, c.seed, c.nheads, st);
  if (e == cudaSuccess)  // empty ring: count = 0 everywhere; zeroed so exports are deterministic
    e = cudaMemsetAsync(x->arena + x->lay.ring_a, 0, x->lay.total - x->lay.ring_a, st);
  if (e == cudaSuccess) e = launch_meta_reset(reinterpret_cast<int4 *>(x->arena + x->lay.meta), c.batch, err_word(x), st);
  if (e != cudaSuccess) return cuda_fail(e);
  x->parity = 0;
  x->loaded = 1;
  x->pos = 0;
  return RSSM_OK;
}

rssm_status rssm_mamba2_step(rssm_ctx *x, const void *xin, const void *B, const void *C, const void *dt, float *y,
                             rssm_stream stream) {
  if (!x) return RSSM_ERR_ARG;
  if (x->cfg.kind != RSSM_MAMBA2) return RSSM_ERR_UNSUPPORTED;
  if (!xin || !B || !C || !dt || !y || !aligned16(xin) || !aligned16(B) || !aligned16(C)) return RSSM_ERR_ARG;
  return run_m2(x, OP_STEP, 1, xin, B, C, dt, nullptr, y, reinterpret_cast<cudaStream_t>(stream));
}

rssm_status rssm_gdn_step(rssm_ctx *x, const void *q, const void *k, const void *v, const float *alpha,
                          const float *beta, float *y, rssm_stream stream) {
  if (!x) return RSSM_ERR_ARG;
  if (x->cfg.kind != RSSM_GDN) return RSSM_ERR_UNSUPPORTED;
  if (!q || !k || !v || !alpha || !beta || !y || !aligned16(q) || !aligned16(k) || !aligned16(v)) return RSSM_ERR_ARG;
  return run_gdn(x, OP_STEP, 1, q, k, v, alpha, beta, nullptr, y, reinterpret_cast<cudaStream_t>(stream));
}

rssm_status rssm_verify(rssm_ctx *x, int T, const rssm_tokens *tok, float *y, rssm_stream stream) {
  if (!x || !tok || !y) return RSSM_ERR_ARG;
  if (T < 1 || T > x->cfg.max_draft) return RSSM_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (x->cfg.kind == RSSM_MAMBA2) {
    if (!tok->x || !tok->B || !tok->C || !tok->dt || !aligned16(tok->x) || !aligned16(tok->B) || !aligned16(tok->C))
      return RSSM_ERR_ARG;
    return run_m2(x, OP_VERIFY, T, tok->x, tok->B, tok->C, tok->dt, nullptr, y, st);
  }
  if (!tok->q || !tok->k || !tok->v || !tok->alpha || !tok->beta || !aligned16(tok->q) || !aligned16(tok->k) ||
      !aligned16(tok->v))
    return RSSM_ERR_ARG;
  return run_gdn(x, OP_VERIFY, T, tok->q, tok->k, tok->v, tok->alpha, tok->beta, nullptr, y, st);
}

rssm_status rssm_commit(rssm_ctx *x, const int *accepted, rssm_stream stream) {
  if (!x || !accepted) return RSSM_ERR_ARG;
  if (!x->loaded) return RSSM_ERR_UNSUPPORTED;
  cudaError_t e = launch_commit(meta_cur(x), meta_next(x), accepted, x->cfg.batch, err_word(x),
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  x->parity ^= 1;
  x->pos = -1;
  return RSSM_OK;
}

rssm_status rssm_flush(rssm_ctx *x, const unsigned char *mask, rssm_stream stream) {
  if (!x) return RSSM_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (x->cfg.kind == RSSM_MAMBA2) return run_m2(x, OP_FLUSH, 0, nullptr, nullptr, nullptr, nullptr, mask, nullptr, st);
  return run_gdn(x, OP_FLUSH, 0, nullptr, nullptr, nullptr, nullptr, nullptr, mask, nullptr, st);
}

rssm_status rssm_export(rssm_ctx *x, float *S_out, void *ring_out, int *meta_out, rssm_stream stream) {
  if (!x) return RSSM_ERR_ARG;
  if (!x->loaded) return RSSM_ERR_UNSUPPORTED;
  const rssm_config &c = x->cfg;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t units = (size_t)c.batch * c.nheads;
  const int esz = esize(c), L = c.window, R = c.headdim;
  cudaError_t e = cudaSuccess;
  if (S_out) {
    if (c.hp == RSSM_HP_F32 && c.read != RSSM_READ_SHARED_NVFP4)
      e = cudaMemcpyAsync(S_out, x->arena + x->lay.hp, units * R * kCols * 4, cudaMemcpyDeviceToDevice, st);
    else
      e = launch_widen_state(x->arena + x->lay.hp, reinterpret_cast<const float *>(x->arena + x->lay.hs), c.hp,
                             x->arena + x->lay.rq, x->arena + x->lay.rs,
                             reinterpret_cast<const float *>(x->arena + x->lay.rg), c.read, S_out, (int)units, R, st);
  }
  if (e == cudaSuccess && meta_out) e = launch_export_meta(meta_cur(x), meta_out, c.batch, L, st);
  if (e == cudaSuccess && ring_out) {
    unsigned char *o = static_cast<unsigned char *>(ring_out);
    const int4 *m = meta_cur(x);
    const int dts = dt_stride(L);
    if (c.kind == RSSM_MAMBA2) {
      e = launch_gather_window(x->arena + x->lay.ring_a, o, m, c.batch, c.nheads, (size_t)2 * L * R * esz, R * esz, L, st);
      o += units * L * R * esz;
      if (e == cudaSuccess)
        e = launch_gather_window(x->arena + x->lay.ring_b, o, m, c.batch, c.ngroups, (size_t)2 * L * kCols * esz,
                                 kCols * esz, L, st);
      o += (size_t)c.batch * c.ngroups * L * kCols * esz;
      if (e == cudaSuccess)
        e = launch_gather_window(x->arena + x->lay.ring_c, o, m, c.batch, c.nheads, (size_t)dts * 4, 4, L, st);
    } else {
      e = launch_gather_window(x->arena + x->lay.ring_a, o, m, c.batch, c.nheads, (size_t)2 * L * kCols * esz,
                               kCols * esz, L, st);
      o += units * L * kCols * esz;
      if (e == cudaSuccess)
        e = launch_gather_window(x->arena + x->lay.ring_b, o, m, c.batch, c.nheads, (size_t)2 * L * R * esz, R * esz, L, st);
      o += units * L * R * esz;
      if (e == cudaSuccess)
        e = launch_gather_window(x->arena + x->lay.ring_c, o, m, c.batch, c.nheads, (size_t)dts * 4, 4, L, st);
      o += units * L * 4;
      if (e == cudaSuccess)
        e = launch_gather_window(x->arena + x->lay.ring_d, o, m, c.batch, c.nheads, (size_t)dts * 4, 4, L, st);
    }
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return RSSM_OK;
}

rssm_status rssm_export_read_copy(rssm_ctx *x, unsigned char *codes, unsigned char *scales, float *g,
                                  rssm_stream stream) {
  if (!x) return RSSM_ERR_ARG;
  const rssm_config &c = x->cfg;
  if (c.read == RSSM_READ_SAME || !x->loaded) return RSSM_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t elems = (size_t)c.batch * c.nheads * c.headdim * kCols;
  cudaError_t e = cudaSuccess;
  if (codes) e = cudaMemcpyAsync(codes, x->arena + x->lay.rq, elems / 2, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && scales) e = cudaMemcpyAsync(scales, x->arena + x->lay.rs, elems / 16, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && g)
    e = cudaMemcpyAsync(g, x->arena + x->lay.rg, (size_t)c.batch * c.nheads * ((c.headdim + 63) / 64) * 4,
                        cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return RSSM_OK;
}

rssm_status rssm_export_column_scales(rssm_ctx *x, unsigned char *colscales, rssm_stream stream) {
  if (!x || !colscales) return RSSM_ERR_ARG;
  const rssm_config &c = x->cfg;
  if (c.read != RSSM_READ_NVFP4D || !x->loaded) return RSSM_ERR_UNSUPPORTED;
  const size_t bytes = (size_t)c.batch * c.nheads * ((c.headdim + 15) / 16) * kCols;
  const cudaError_t e = cudaMemcpyAsync(colscales, x->arena + x->lay.rc, bytes, cudaMemcpyDeviceToDevice,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_export_skip(rssm_ctx *x, unsigned char *flags, rssm_stream stream) {
  if (!x || !flags) return RSSM_ERR_ARG;
  if (!x->loaded || x->cfg.skip_tau == 0.f) return RSSM_ERR_UNSUPPORTED;
  const size_t units = (size_t)x->cfg.batch * x->cfg.nheads;
  cudaError_t e = cudaMemcpyAsync(flags, x->arena + x->lay.skip, units, cudaMemcpyDeviceToDevice,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_get_error(rssm_ctx *x, int *code, int *seq, rssm_stream stream) {
  if (!x || !code || !seq) return RSSM_ERR_ARG;
  if (!x->loaded) return RSSM_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int w = kErrClean;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&w, err_word(x), sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (w == kErrClean) {
    *code = RSSM_DEV_OK;
    *seq = -1;
    return RSSM_OK;
  }
  *code = w & 15;
  *seq = w >> 4;
  return RSSM_ERR_DEVICE;
}

// ------------------------------------------------------------------ comparison kernels

static rssm_status conv_common(const rssm_config *cfg, ConvArgs &a) {
  if (!cfg) return RSSM_ERR_ARG;
  rssm_config c = *cfg;
  c.hp = RSSM_HP_F32;
  c.read = RSSM_READ_SAME;
  rssm_status s = validate(&c);
  if (s != RSSM_OK) return s;
  a.kind = c.kind; a.Bt = c.batch; a.H = c.nheads; a.R = c.headdim; a.G = c.ngroups;
  a.q_scale = c.q_scale; a.A = c.A; a.D = c.D;
  return RSSM_OK;
}

rssm_status rssm_conv_mamba2_step(const rssm_config *cfg, float *S, const void *xin, const void *B, const void *C,
                                  const void *dt, float *y, rssm_stream stream) {
  ConvArgs a{};
  rssm_status s = conv_common(cfg, a);
  if (s != RSSM_OK) return s;
  if (cfg->kind != RSSM_MAMBA2) return RSSM_ERR_UNSUPPORTED;
  if (!S || !xin || !B || !C || !dt || !y || !aligned16(S) || !aligned16(xin) || !aligned16(B) || !aligned16(C))
    return RSSM_ERR_ARG;
  a.T = 1; a.tmax = 0; a.S = S; a.x = xin; a.Bin = B; a.C = C; a.dt = dt; a.y = y;
  cudaError_t e = launch_conv(a, esize(*cfg), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_conv_gdn_step(const rssm_config *cfg, float *S, const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta, float *y, rssm_stream stream) {
  ConvArgs a{};
  rssm_status s = conv_common(cfg, a);
  if (s != RSSM_OK) return s;
  if (cfg->kind != RSSM_GDN) return RSSM_ERR_UNSUPPORTED;
  if (!S || !q || !k || !v || !alpha || !beta || !y || !aligned16(S) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return RSSM_ERR_ARG;
  a.T = 1; a.tmax = 0; a.S = S; a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.y = y;
  cudaError_t e = launch_conv(a, esize(*cfg), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_snap_verify(const rssm_config *cfg, float *snaps, const int *cur, int T, const rssm_tokens *tok,
                             float *y, rssm_stream stream) {
  ConvArgs a{};
  rssm_status s = conv_common(cfg, a);
  if (s != RSSM_OK) return s;
  if (!snaps || !cur || !tok || !y || !aligned16(snaps)) return RSSM_ERR_ARG;
  if (T < 1 || T > cfg->max_draft) return RSSM_ERR_ARG;
  a.T = T; a.tmax = cfg->max_draft; a.S = snaps; a.cur = cur; a.y = y;
  if (cfg->kind == RSSM_MAMBA2) {
    if (!tok->x || !tok->B || !tok->C || !tok->dt || !aligned16(tok->x) || !aligned16(tok->B) || !aligned16(tok->C))
      return RSSM_ERR_ARG;
    a.x = tok->x; a.Bin = tok->B; a.C = tok->C; a.dt = tok->dt;
  } else {
    if (!tok->q || !tok->k || !tok->v || !tok->alpha || !tok->beta || !aligned16(tok->q) || !aligned16(tok->k) ||
        !aligned16(tok->v))
      return RSSM_ERR_ARG;
    a.q = tok->q; a.k = tok->k; a.v = tok->v; a.alpha = tok->alpha; a.beta = tok->beta;
  }
  cudaError_t e = launch_conv(a, esize(*cfg), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_snap_commit(const rssm_config *cfg, int *cur, const int *accepted, rssm_stream stream) {
  if (!cfg || !cur || !accepted) return RSSM_ERR_ARG;
  if (cfg->batch < 1 || cfg->max_draft < 1) return RSSM_ERR_SHAPE;
  cudaError_t e = launch_snap_commit(cur, accepted, cfg->batch, cfg->max_draft + 1, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

rssm_status rssm_sched_probe(int units, int blocks, int *per_block, int *bad_units, rssm_stream stream) {
  if (units < 1 || units > kProbeMaxUnits || blocks < 1 || blocks > kProbeMaxBlocks || !per_block || !bad_units)
    return RSSM_ERR_ARG;
  const cudaError_t e = launch_sched_probe(units, blocks, per_block, bad_units, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSSM_OK : cuda_fail(e);
}

}  // extern "C"
