// common.cuh -- device helpers shared by the ReplaySSM kernels (sm_100a).
//
// * mbarrier + cp.async.bulk (TMA bulk copy, global -> shared) primitives used by
//   the persistent streaming kernels: one producer warp issues bulk copies of a
//   head's checkpoint tile and its buffered inputs into a shared-memory stage,
//   consumer warps wait on the stage's "full" barrier and release it through an
//   "empty" barrier.  Every wait is bounded: after ~1 s of polling it records
//   RSSM_DEV_TIMEOUT in the context's error word and the kernel winds down.
// * warp-level transpose reduction: each lane holds V partial sums; after
//   log2(32) exchange levels every value has been summed over the 32 lanes and
//   each lane keeps max(V/32, 1) of them (lane l keeps indices l*V/32 + i).
// * arena layout shared by the host API and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rssm.h"

namespace rssm {

constexpr int kCols = 128;           // contiguous state axis (N or d_k)
constexpr int kMaxWindow = 32;
constexpr int kMaxDraft = 8;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + one producer warp
constexpr long long kWaitCycles = 2000000000LL;  // default bound of every wait, ~1 s at B200 clocks
constexpr unsigned int kSuspendNs = 0;           // default suspend-time hint of a barrier poll (hardware default)

// error word: min over (seq * 16 + code); 0x7fffffff = clean
constexpr int kErrClean = 0x7fffffff;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
__host__ __device__ inline int dt_stride(int L) { return (int)align_up((size_t)(2 * L), 4); }  // fp32 slots per ring row

// Byte offsets of the regions of a context's arena.
struct ArenaLayout {
  size_t meta;     // int4 [2][Bt]: count, epoch, pending, 0  (ping-pong by call parity)
  size_t err;      // int [4]: sticky error word, next unit to hand out, blocks finished, 0
  size_t hp;       // checkpoint: fp32, fp16 or E4M3 [Bt][H][R][128]
  size_t hs;       // E4M3 checkpoint tile scales fp32 [Bt][H][ceil(R/64)] (padded to 16 bytes)
  size_t rq;       // NVFP4 codes u8 [Bt][H][R][64]
  size_t rs;       // NVFP4 block scales u8 [Bt][H][R][8]
  size_t rg;       // NVFP4 tile scale fp32 [Bt][H][ceil(R/64)] (padded to 16 bytes)
  size_t rc;       // two-axis copy: column-group scales u8 [Bt][H][ceil(R/16)][128]
  size_t ring_a;   // Mamba-2 x [Bt][H][2L][P] / GDN k [Bt][H][2L][128]   (input dtype)
  size_t ring_b;   // Mamba-2 B [Bt][G][2L][128] / GDN v [Bt][H][2L][d_v] (input dtype)
  size_t ring_c;   // Mamba-2 dt / GDN alpha: fp32 [Bt][H][dt_stride(L)]
  size_t ring_d;   // GDN beta: fp32 [Bt][H][dt_stride(L)]
  size_t skip;     // decay-aware skip flags u8 [Bt][H] (only with skip_tau > 0)
  size_t total;
};

inline ArenaLayout make_layout(const rssm_config &c) {
  ArenaLayout a{};
  const size_t Bt = c.batch, H = c.nheads, R = c.headdim, L = c.window;
  const size_t esz = c.in_dtype == RSSM_BF16 ? 2 : 4;
  const size_t units = Bt * H;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  a.meta = take(2 * Bt * 16);
  a.err = take(16);
  const bool shared_fp4 = c.read == RSSM_READ_SHARED_NVFP4;
  const size_t hp_esz = c.hp == RSSM_HP_F16_SR ? 2 : c.hp == RSSM_HP_F8_SR ? 1 : 4;
  a.hp = take(shared_fp4 ? 0 : units * R * kCols * hp_esz);
  a.hs = take(!shared_fp4 && c.hp == RSSM_HP_F8_SR ? align_up(units * ((R + 63) / 64), 4) * 4 : 0);
  const bool fp4 = c.read != RSSM_READ_SAME;
  a.rq = take(fp4 ? units * R * kCols / 2 : 0);
  a.rs = take(fp4 ? units * R * kCols / 16 : 0);
  const size_t nrb = (R + 63) / 64;  // NVFP4 tiles (64-row blocks) per head
  a.rg = take(fp4 ? align_up(units * nrb, 4) * 4 : 0);
  a.rc = take(c.read == RSSM_READ_NVFP4D ? units * ((R + 15) / 16) * kCols : 0);
  if (c.kind == RSSM_MAMBA2) {
    a.ring_a = take(units * 2 * L * R * esz);
    a.ring_b = take(Bt * c.ngroups * 2 * L * kCols * esz);
    a.ring_c = take(units * dt_stride(c.window) * 4);
    a.ring_d = take(0);
  } else {
    a.ring_a = take(units * 2 * L * kCols * esz);
    a.ring_b = take(units * 2 * L * R * esz);
    a.ring_c = take(units * dt_stride(c.window) * 4);
    a.ring_d = take(units * dt_stride(c.window) * 4);
  }
  a.skip = take(c.skip_tau > 0.f ? units : 0);
  a.total = off;
  return a;
}

// ------------------------------------------------------------------------------------------
// loads / conversions

__device__ __forceinline__ float4 f4zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// 4 consecutive elements starting at p (16-byte aligned for float, 8-byte for bf16)
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  float4 r;
  r.x = __uint_as_float(u.x << 16);
  r.y = __uint_as_float(u.x & 0xffff0000u);
  r.z = __uint_as_float(u.y << 16);
  r.w = __uint_as_float(u.y & 0xffff0000u);
  return r;
}

// 8 consecutive elements starting at p (16-byte aligned for bf16, 32-byte for float)
__device__ __forceinline__ void load8(const float *p, float (&o)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&o)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  o[0] = __uint_as_float(u.x << 16); o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16); o[3] = __uint_as_float(u.y & 0xffff0000u);
  o[4] = __uint_as_float(u.z << 16); o[5] = __uint_as_float(u.z & 0xffff0000u);
  o[6] = __uint_as_float(u.w << 16); o[7] = __uint_as_float(u.w & 0xffff0000u);
}

__device__ __forceinline__ void record_error(int *err, int seq, int code) { atomicMin(err, seq * 16 + code); }

// ------------------------------------------------------------------------------------------
// mbarrier / bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// How a wait spins: `limit` clock cycles in all, and each try_wait may suspend the warp for up to
// `hint_ns` nanoseconds until the phase completes (0: the hardware's default), so that waiting warps
// take fewer issue slots from working ones.
struct WaitSpec {
  long long limit;
  uint32_t hint_ns;
};

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  if (hint_ns)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity: false after ws.limit clock cycles.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, WaitSpec ws) {
  if (mbar_try_wait(bar, parity, ws.hint_ns)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity, ws.hint_ns)) {
    if (clock64() - t0 > ws.limit) return false;
  }
  return true;
}

// Bounded wait that also gives up as soon as another warp of the block has flagged an abort.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                   WaitSpec ws) {
  if (mbar_try_wait(bar, parity, ws.hint_ns)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity, ws.hint_ns)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > ws.limit) return false;
  }
  return true;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// global -> shared bulk copy completing on an mbarrier; dst, src 16-byte aligned, bytes % 16 == 0
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// shared -> global bulk copy (TMA store), tracked by the issuing thread's bulk async-group
__device__ __forceinline__ void bulk_s2g(void *gdst, const void *ssrc, uint32_t bytes, uint64_t policy) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until the committed bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until the committed bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// make this thread's generic-proxy shared-memory writes visible to the async proxy (bulk copies)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// consumer-only named barrier (the producer warp does not take part)
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

// ------------------------------------------------------------------------------------------
// warp reductions

template <int V>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[V], int lane) {
  int cur = V;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (cur > 1) {
      const int half = cur / 2;
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < half) {
          float send = upper ? v[i] : v[i + half];
          float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      cur = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

// ---- dynamic unit scheduling.  A launch hands its work units to its persistent blocks through a
// counter next to the error word (one atomic per unit), so that blocks whose units cost more (a fold
// reads and writes the state) do not hold up a launch whose other blocks drew cheaper ones.  The last
// block to finish re-arms the counters for the next launch on the stream.
__device__ __forceinline__ int sched_grab(int *err) { return atomicAdd(err + 1, 1); }
__device__ __forceinline__ void sched_finish(int *err) {  // one thread per block, after the block's last grab
  if (atomicAdd(err + 2, 1) == (int)gridDim.x - 1) {
    atomicExch(err + 1, 0);
    atomicExch(err + 2, 0);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// four 8x8 b16 matrices from shared memory; lane l gives the (16-byte aligned) address of row l & 7 of
// matrix l >> 3, and register q of lane 4g+t receives elements 2t, 2t+1 of row g of matrix q
__device__ __forceinline__ void ldmatrix_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p))
               : "memory");
}

// the same with each 8x8 matrix transposed: register q of lane 4g+t receives rows 2t, 2t+1 of column g
__device__ __forceinline__ void ldmatrix_x4_trans(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                                  uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p))
               : "memory");
}

// ---- register-operand tensor-core tile (warp-wide): d[16x8] += a[16x16] b[16x8], bf16 in, fp32 accumulate.
// Lane 4g+t holds a = {A[g][2t..2t+1], A[g+8][2t..2t+1], A[g][2t+8..2t+9], A[g+8][2t+8..2t+9]},
// b = {B[2t..2t+1][g], B[2t+8..2t+9][g]}, d = {D[g][2t..2t+1], D[g+8][2t..2t+1]}; the lower-indexed
// element of a pair sits in the low half of its register.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp32 pair -> bf16 pairs hi + lo with hi = RN(v) and lo = RN(v - hi): |v - hi - lo| <= 2^-17 |v|, so two
// bf16 products against an exact bf16 operand carry a fp32 operand to ~16 significant bits.
__device__ __forceinline__ void split_bf16x2(float x, float y, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const uint32_t hb = *reinterpret_cast<const uint32_t *>(&h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - __uint_as_float(hb << 16), y - __uint_as_float(hb & 0xffff0000u));
  hi = hb;
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// fp32 pair -> bf16 pairs hi + mid + lo, each piece the leading 16 bits of what the previous ones left.
// The split is exact: a fp32 significand has 24 bits, each piece takes the leading 8 of the remainder,
// and the subtractions x - piece are exact, so hi + mid + lo == x.
__device__ __forceinline__ void split3_bf16x2(float x, float y, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
  const uint32_t xb = __float_as_uint(x), yb = __float_as_uint(y);
  hi = __byte_perm(xb, yb, 0x7632);
  const float x1 = x - __uint_as_float(xb & 0xffff0000u), y1 = y - __uint_as_float(yb & 0xffff0000u);
  const uint32_t x1b = __float_as_uint(x1), y1b = __float_as_uint(y1);
  mid = __byte_perm(x1b, y1b, 0x7632);
  const float x2 = x1 - __uint_as_float(x1b & 0xffff0000u), y2 = y1 - __uint_as_float(y1b & 0xffff0000u);
  lo = __byte_perm(__float_as_uint(x2), __float_as_uint(y2), 0x7632);
}

}  // namespace rssm
