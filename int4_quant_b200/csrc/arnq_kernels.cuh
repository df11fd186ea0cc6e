// arnq_kernels.cuh -- sm_100a kernels for the fused residual add + RMSNorm +
// per-row symmetric dynamic quantization operator (CANN page
// "aclnnAddRmsNormDynamicQuantV2", section "Formula"; the no-add form is the
// page "aclnnRmsNormDynamicQuant", formula section).
//
// One kernel template, three ways of bringing a row on chip:
//   LOAD_VEC     16-byte vector loads straight into registers (8 elements a unit)
//   LOAD_SCALAR  2-byte loads of element pairs, for misaligned tensors or n % 8 != 0
//   LOAD_STAGED  one thread copies the CTA's slice of upcoming rows into shared
//                memory with cp.async.bulk (1-D bulk copies completing on an
//                mbarrier); a ring of `stages` rows keeps HBM reads in flight
//                while the threads work on the current row.
// A CTA (or, for rows too long for one CTA or too few rows to fill the SMs, a
// thread-block cluster of CTAs sharing a row through distributed shared memory)
// takes one row at a time; each thread keeps its elements of x and its folded
// parameters G_k in registers (B_k of 16-byte units in shared memory, read
// back by the thread that wrote it).  Persistent grid: a CTA takes rows c,
// c + G, ... and then (staged kernel, one CTA per row) rows handed out one at
// a time by a counter in the workspace.  Three barriers per row: after the
// sum of squares, after the binary32 row maxima and after the exact row
// maxima.  The kernel is launched as a programmatic dependent (it waits for
// the preceding work before touching memory, and lets the next kernel start
// its set-up after its last row).
//
// The result is what an fp64 evaluation of the definition gives, with the
// scale rounded to binary32: scale_k = RN32(max|input_k| / Q) and
// code = RNE(input_k / scale_k).  Per row:
//   x = RN16(x1 + x2)            add.rn.{bf16,f16}x2 -- the correctly rounded
//                                sum, which equals rounding the binary32 sum;
//                                written as xOut and kept in registers
//   ss = sum x^2                 fp64 (each x^2 is exact)
//   1/Rms                        binary32 from ss (within a few ulp)
//   input_k = x*rinv*G_k + B_k   binary32, packed f32x2 (add/mul/fma.rn.f32x2);
//                                G_k = gamma*smooth_k, B_k = beta*smooth_k,
//                                exact products of two 16-bit values
//   max_k                        binary32 row maximum, then exact: the threads
//                                holding a candidate unit (an element within
//                                the binary32 error bound of that maximum; the
//                                true maximum is among them) evaluate its
//                                elements in fp64, and the fp64 maxima meet
//                                at the third barrier
//   scale_k = RN32(max_k / Q)    exact
//   code = RNE(input_k * RN32(1/scale_k))  binary32, rounded half to even by
//                                adding 1.5*2^23; a code whose quotient lies
//                                within tau of a half-way point (tau bounds the
//                                binary32 error) is recomputed by its thread in
//                                fp64 as input_k / scale_k (about 1e-3 of the
//                                codes)
// The fp64 inputs use 1/Rms from Newton steps (a few fp64 ulp): the decisions
// they settle sit many orders of magnitude above fp64 rounding.  A row whose
// ss/n + eps leaves the normal binary32 range is computed whole in fp64, in
// the definition's order with IEEE divisions; one whose 1/scale is not a
// normal binary32 number gets all its codes in fp64.  Every thread handles
// its own elements: no global memory is read twice.
// Nothing here is a contraction: no tensor cores.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace arnq {
namespace cg = cooperative_groups;

enum : int {
  F_BETA = 1,   // beta given
  F_XOUT = 2    // xOut written
};
enum : int { LOAD_VEC = 0, LOAD_SCALAR = 1, LOAD_STAGED = 2 };

// status codes the kernels record in the workspace status block
enum : int {
  DEV_TIMEOUT = 11,   // a bounded wait ran out
  DEV_SCHED = 12      // the row hand-out counters were not zero when the call started
};

// A bounded wait gives up after this long (nanoseconds of %globaltimer)
// unless the launch asks for another limit.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// row flags exchanged at the first barrier of the next row
enum : int { RF_REDO = 1, RF_ABORT = 2 };

// The workspace holds only the status block (kStatusBytes: the status at
// bytes 0-15, the row hand-out counters at 16-27).
constexpr int kStatusBytes = 256;

// Row records.  The binary32 fast path leaves a few units (8 or 2 elements)
// per row that it cannot settle: candidate units, holding an element within
// the binary32 error bound of the row maximum (the true maximum is among
// them), and near-tie units, holding a code whose binary32 quotient lies
// within tau of a half-way point.  The thread that holds such a unit appends
// it to the row's record together with the unit's G_k and B_k; one row later
// one warp (the settling warp) copies the recorded units' x from xOut (or
// x1, x2) into the record with cp.async, and one row later again settles the
// row from the record alone: the exact scale RN32(max fp64 |input| over the
// candidates / Q), then the near-tie codes in fp64 -- with no load on its
// critical path.  Three records live in the shared memory of the row's CTA
// (of the cluster's first CTA): the row being processed, the one whose x is
// on its way, and the one being settled.
//   header (32 B): double ss; int cnt[2] (candidate, near-tie entries); int flags
//   ue  [cap] ints: unit | output << 31, candidates first (cap = kCandCap + tie_cap)
//   ent [cap][24] 32-bit words: x (16 bytes: eight 16-bit values, or x1 then
//       x2 when xOut is not written; 32 bytes reserved), G_k (8 floats), B_k
//       (8 floats); pair units (2 elements) use the first words of each part
// A row whose near-tie list overflows (many exact ties) or whose arithmetic
// leaves the normal binary32 range is recomputed whole, in fp64.
constexpr int kCandCap = 4;
__host__ __device__ inline int tie_cap(int n, int nout) { return 12 + (n * nout + 255) / 256; }
struct RecHead {
  double ss;
  int cnt[2];
  int flags;
  int pad[3];
};
__host__ __device__ inline int rec_ue_bytes(int tcap) { return ((kCandCap + tcap) * 4 + 15) & ~15; }
__host__ __device__ inline int rec_slot_bytes(int tcap) {
  return static_cast<int>(sizeof(RecHead)) + rec_ue_bytes(tcap) + (kCandCap + tcap) * 96;
}

// Shared-memory layout, sized by the launch (the host computes the same):
//   ss    [nslots] doubles: per-warp partial sums (also the exact path's reductions)
//   wmax  [NOUT][nslots] floats: per-warp binary32 row maxima of |input_k|
//   maxb  [NOUT][nslots] floats: set-up reduction of the bound on |B_k|
//   flags [2] ints: RF_* of a row, by row parity
//   bars  [stages] mbarriers
//   recs  [3] row records of rec_bytes each (used in the cluster's first CTA)
//   srow  [stages] int64: staged kernel, the row each stage holds (-1: none)
//   take  16 bytes: the copy-issuing thread's row hand-out state (TakeState)
//   bsm   16-byte units: B_k = beta * smooth_k of every thread's units,
//         [NOUT][UPT][2][threads] float4 (bsm_bytes_for)
//   ring  [stages] rows of staged input
// nslots = warps per CTA times CTAs per cluster.
constexpr int kMaxStagesDev = 8;
// shared memory holding B_k for a CTA of `threads` threads, `upt` 16-byte units
// each (0 for 2-element units, whose B_k stay in registers)
__host__ __device__ inline int bsm_bytes_for(bool vector_units, int nout, int upt, int threads) {
  return vector_units ? nout * upt * threads * 32 : 0;
}
struct Layout {
  int ss, wmax, maxb, flags, bars, srow, take, recs, bsm, ring;
};
struct TakeState {
  int64_t nxt;   // next row dealt out in turn
  int ndyn;      // rows taken from the counter
  int dry;       // the counter ran out: take nothing more
};
__host__ __device__ inline Layout make_layout(int nslots, int nout, int stages, int rec_bytes,
                                              int bsm_bytes) {
  Layout L;
  int off = 0;
  L.ss = off;    off += nslots * 8;
  L.wmax = off;  off += nout * nslots * 4;
  L.maxb = off;  off += nout * nslots * 4;
  off = (off + 7) & ~7;
  L.flags = off; off += 2 * 4;
  off = (off + 7) & ~7;
  L.bars = off;  off += stages * 8;
  L.srow = off;  off += stages * 8;
  L.take = off;  off += 16;
  off = (off + 15) & ~15;
  L.recs = off;  off += 3 * rec_bytes;
  off = (off + 15) & ~15;
  L.bsm = off;   off += bsm_bytes;
  L.ring = (off + 127) & ~127;
  return L;
}

struct KParams {
  const uint16_t *x1, *x2, *gamma, *beta;
  const uint16_t *smooth[2];  // per output slot; nullptr = no smooth scale
  uint8_t *y[2];              // per output slot
  float *scale[2];            // per output slot
  uint16_t *x_out;
  int32_t *status;            // workspace status block
  int32_t *sched;             // workspace: tickets handed out, CTAs done, rows handed out
                              // (all zero between calls)
  int64_t dyn_base;           // staged, one CTA per row: rows from here on are handed
                              // out by the counter (rows = none)
  int64_t rows;
  int32_t n;                  // row length in elements
  int32_t units;              // units per row: ceil(n / U)
  int32_t seg_units;          // units per CTA of a cluster
  int32_t flags;
  int32_t stages;             // staged kernel: ring depth
  int32_t tie_cap;            // near-tie entries a record holds
  int32_t rec_bytes;          // bytes of one record (rec_slot_bytes)
  float eps;
  double inv_n;               // 1 / n
  uint64_t wait_limit_ns;     // bounded waits give up after this long
  uint32_t test_hold_tx;      // testing only: extra bytes the first staged copy's
                              // barrier expects (never delivered); 0 in normal use
};

struct Bf16 {};
struct Fp16 {};

template <class T> struct Cvt;
template <> struct Cvt<Bf16> {
  // two packed bf16 -> two floats (exact: a bf16 is the top half of a binary32)
  static __device__ __forceinline__ float2 f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  static __device__ __forceinline__ float f1(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  // two floats -> two packed bf16, round to nearest even (cvt.rn.bf16x2.f32)
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    uint32_t w;
    memcpy(&w, &h, 4);
    return w;
  }
  // correctly rounded sum of two packed pairs.  The binary32 sum of two bf16
  // values is exact unless their exponents differ by more than 16, and then the
  // smaller one is below half an ulp of the result and cannot move a rounding
  // decision: RN16(a + b) == RN16(RN32(a + b)).
  static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
  }
};
template <> struct Cvt<Fp16> {
  static __device__ __forceinline__ float2 f2(uint32_t w) {
    __half2 h;
    memcpy(&h, &w, 4);
    return __half22float2(h);
  }
  static __device__ __forceinline__ float f1(uint16_t u) {
    __half h;
    memcpy(&h, &u, 2);
    return __half2float(h);
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    uint32_t w;
    memcpy(&w, &h, 4);
    return w;
  }
  // as for bf16: the binary32 sum of two fp16 values is exact unless the
  // exponents differ by more than 13, when the smaller is below half an ulp.
  static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
  }
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// One try of an mbarrier phase wait; the thread may sleep in hardware for up
// to kSuspendHintNs while the phase is incomplete.
constexpr uint32_t kSuspendHintNs = 100000u;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Waits for the given phase parity of an mbarrier, at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16; `policy` an L2 cache policy.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// 16-byte copy global -> shared (cp.async, through L2 only); completes for
// the issuing thread at cp.async.wait_group
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// L2 policy of the staged input copies: normal eviction (measured faster than
// evict-first on the 8192 x 4096 workload, where x1, x2 and the outputs
// together exceed L2).
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}


// 16-byte streaming load (read once: evict-first in L1 and L2).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  return __ldcs(reinterpret_cast<const uint4 *>(p));
}
// 16-byte read-only load for parameters (kept in cache).
__device__ __forceinline__ uint4 ld_param16(const void *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
// max over lanes of non-negative floats (their bit patterns order as integers)
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v)));
}

// 1/sqrt(v) in binary32: the hardware estimate refined by one Newton-Raphson
// step, r' = r (3 - v r^2) / 2; within 3 ulp.
__device__ __forceinline__ float rsqrt_refined(float v) {
  const float r = rsqrtf(v);
  const float h = 0.5f * v;
  return r * __fmaf_rn(-h * r, r, 1.5f);
}

// Threads per CTA the register budget allows.  A thread keeps, per element, x
// and per output G and B: (1 + 2*NOUT) floats.  Up to 48 of them fit the 64
// registers of a 1024-thread CTA, up to 112 the 128 of 512 threads; more get 255.
__host__ __device__ constexpr int max_threads_for(int mode, int upt, int nout) {
  return (upt * (mode == LOAD_SCALAR ? 2 : 8) * (1 + 2 * nout) <= 48)    ? 1024
         : (upt * (mode == LOAD_SCALAR ? 2 : 8) * (1 + 2 * nout) <= 112) ? 512
                                                                         : 256;
}

constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: v + kMagic = RNE(v) + kMagic
constexpr float kUnit = 5.9604644775390625e-08f;  // 2^-24, binary32 unit roundoff

// ------------------------------------------------------- exact (fp64) pieces

// 1/sqrt(v) in fp64 to a few ulp, for v in the normal binary32 range: the
// binary32 estimate refined by two Newton steps r' = r + r(1 - v r^2)/2.
__device__ __forceinline__ double rsqrt64(double v) {
  double r = static_cast<double>(rsqrtf(__double2float_rn(v)));
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const double e = __fma_rn(-__dmul_rn(v, r), r, 1.0);
    r = __fma_rn(__dmul_rn(0.5, r), e, r);
  }
  return r;
}
// round half to even, clamped to [-qmax, qmax]
__device__ __forceinline__ int code_of_t(double t, int qmax) {
  return min(max(__double2int_rn(t), -qmax), qmax);
}

// In the definition's order with IEEE-rounded fp64 operations (the slow path):
//   Rms = sqrt(ss / n + eps);  y = x / Rms * gamma (+ beta);  input = y (* smooth)
__device__ __forceinline__ double rms_of(double ss, int n, float eps) {
  return __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(n)), static_cast<double>(eps)));
}

template <class T>
__device__ __forceinline__ double input_of(const KParams &p, int o, int c, float x, double rms) {
  double y = __dmul_rn(__ddiv_rn(static_cast<double>(x), rms),
                       static_cast<double>(Cvt<T>::f1(__ldg(p.gamma + c))));
  if (p.flags & F_BETA) y = __dadd_rn(y, static_cast<double>(Cvt<T>::f1(__ldg(p.beta + c))));
  if (p.smooth[o]) y = __dmul_rn(y, static_cast<double>(Cvt<T>::f1(__ldg(p.smooth[o] + c))));
  return y;
}

// round_half_even(input / scale) clamped to [-qmax, qmax]; 0 for a zero scale
__device__ __forceinline__ int code_of(double in, float scale, int qmax) {
  if (scale == 0.f) return 0;
  return code_of_t(__ddiv_rn(in, static_cast<double>(scale)), qmax);
}

// ---------------------------------------------------------------- exact codes

// RNE(in / sc) clamped to [-qmax, qmax], for an fp64 input `in`, a positive
// normal binary32 scale sc and an approximation t of in / sc that is off by
// less than 1/2: the only rounding boundary within reach is the half-integer
// h = floor(t) + 1/2, and the sign of in - h*sc decides on which side of it
// in / sc lies.  h*sc is exact in fp64 (a half-integer of at most 9 bits
// times a 24-bit significand), so the fused multiply-add computes that sign
// exactly: the code is correctly rounded, exact ties to even included, with
// no division.
__device__ __forceinline__ int code_exact(double in, float sc, float t, int qmax) {
  const float h = floorf(t) + 0.5f;
  const double e = __fma_rn(-static_cast<double>(h), static_cast<double>(sc), in);
  const int lo = static_cast<int>(h - 0.5f);  // floor(t)
  int q;
  if (e > 0.0) q = lo + 1;
  else if (e < 0.0) q = lo;
  else q = (lo & 1) ? lo + 1 : lo;  // an exact tie: to even
  return min(max(q, -qmax), qmax);
}

// ---------------------------------------------------------------- whole rows in fp64

// x of column c of a row, read back from memory: xOut when written, else the
// inputs (then unchanged: an in-place update always writes xOut).
template <class T, bool ADD>
__device__ __forceinline__ float x_reload(const KParams &p, int64_t row, int c) {
  using C = Cvt<T>;
  const int64_t j = row * p.n + c;
  if (!ADD) return C::f1(p.x1[j]);
  if (p.flags & F_XOUT) return C::f1(p.x_out[j]);
  return C::f2(C::add2(p.x1[j], p.x2[j])).x;
}

// Whole row in fp64, in the definition's order with IEEE divisions, by the 32
// lanes of a warp, x read back from memory: the slow path for rows the fast
// path cannot settle (a near-tie list that overflowed, or ss/n + eps or the
// scale outside the normal binary32 range).  Called, not inlined: rare, and
// its division sequences would take registers from the row loop.
template <class T, bool INT4, int NOUT, bool ADD>
__device__ __noinline__ void exact_row_warp(const KParams &p, int64_t row, int lane) {
  constexpr int QI = INT4 ? 7 : 127;
  const int n = p.n;
  const int64_t base = row * n;
  double ss = 0.0;
  for (int c = lane; c < n; c += 32) {
    const double a = x_reload<T, ADD>(p, row, c);
    ss = __fma_rn(a, a, ss);
  }
  const double rms = rms_of(warp_sum_d(ss), n, p.eps);
  for (int o = 0; o < NOUT; ++o) {
    double m = 0.0;
    for (int c = lane; c < n; c += 32)
      m = fmax(m, fabs(input_of<T>(p, o, c, x_reload<T, ADD>(p, row, c), rms)));
    const float sc = __double2float_rn(__ddiv_rn(warp_max_d(m), static_cast<double>(QI)));
    if (lane == 0) p.scale[o][row] = sc;
    for (int c = 2 * lane; c < n; c += 64) {  // element pairs: an INT4 byte has one writer
      const int q0 = code_of(input_of<T>(p, o, c, x_reload<T, ADD>(p, row, c), rms), sc, QI);
      const int q1 =
          c + 1 < n ? code_of(input_of<T>(p, o, c + 1, x_reload<T, ADD>(p, row, c + 1), rms), sc, QI)
                    : 0;
      if (INT4) {
        p.y[o][row * (n / 2) + c / 2] = static_cast<uint8_t>((q0 & 0xF) | ((q1 & 0xF) << 4));
      } else {
        p.y[o][base + c] = static_cast<uint8_t>(q0);
        if (c + 1 < n) p.y[o][base + c + 1] = static_cast<uint8_t>(q1);
      }
    }
  }
}

// ---------------------------------------------------------------- settling a record

__device__ __forceinline__ int *rec_ue(RecHead *h) { return reinterpret_cast<int *>(h + 1); }
__device__ __forceinline__ uint32_t *rec_ent(RecHead *h, int tcap, int ent) {
  return reinterpret_cast<uint32_t *>(reinterpret_cast<unsigned char *>(h + 1) +
                                      rec_ue_bytes(tcap)) + ent * 24;
}

// Copies the recorded units' x of row r into the record h (16-byte units:
// cp.async, one commit group per call, waited for by the same warp at the
// row's settle).  Rows the slow path takes need nothing.
template <bool ADD, int U>
__device__ __forceinline__ void prefetch_record(const KParams &p, RecHead *h, int64_t r, int lane) {
  if (U == 8) {
    const int nc = min(h->cnt[0], kCandCap), nt = min(h->cnt[1], p.tie_cap);
    const int *ue = rec_ue(h);
    for (int q = lane; q < kCandCap + nt; q += 32) {
      if (q >= nc && q < kCandCap) continue;
      const int u = static_cast<int>(static_cast<uint32_t>(ue[q]) & 0x7FFFFFFFu);
      const int64_t j = r * p.n + static_cast<int64_t>(u) * 8;
      uint32_t *dst = rec_ent(h, p.tie_cap, q);
      if (!ADD) {
        cp_async16(dst, p.x1 + j);
      } else if (p.flags & F_XOUT) {
        cp_async16(dst, p.x_out + j);
      } else {
        cp_async16(dst, p.x1 + j);
        cp_async16(dst + 4, p.x2 + j);
      }
    }
  }
  cp_async_commit();
}

// Settles row r from its record h (in this CTA's shared memory, or the
// cluster's first CTA's) with one warp, then clears the record's counters.
// The record holds every value needed (x copied in by prefetch_record, whose
// group the caller has waited for; G_k and B_k from the recording threads):
// the candidates' fp64 maximum gives the exact scale RN32(max / Q); each
// near-tie unit's codes are then decided exactly from their fp64 inputs
// (code_exact).  Pair units (U == 2: misaligned or ragged rows) read x from
// memory here.
template <class T, bool INT4, int NOUT, bool ADD, int U>
__device__ __forceinline__ void settle_record(const KParams &p, RecHead *h, int64_t r, int lane) {
  using C = Cvt<T>;
  constexpr int QI = INT4 ? 7 : 127;
  constexpr int PAIRS = U / 2;
  const int n = p.n;
  const int nc = h->cnt[0], nt = h->cnt[1];
  if ((h->flags & RF_REDO) || nc > kCandCap || nt > p.tie_cap) {
    exact_row_warp<T, INT4, NOUT, ADD>(p, r, lane);
  } else {
    const int *ue = rec_ue(h);
    const double ri = rsqrt64(__fma_rn(h->ss, p.inv_n, static_cast<double>(p.eps)));
    // fp64 input of element e of entry ent (column c)
    auto in64 = [&](int ent, int e, int c) -> double {
      const uint32_t *v = rec_ent(h, p.tie_cap, ent);
      float x;
      if (U == 8) {
        const int wd = e >> 1;
        const float2 a = C::f2(ADD && !(p.flags & F_XOUT) ? C::add2(v[wd], v[4 + wd]) : v[wd]);
        x = (e & 1) ? a.y : a.x;
      } else {
        x = x_reload<T, ADD>(p, r, c);
      }
      return __fma_rn(__dmul_rn(static_cast<double>(x), ri),
                      static_cast<double>(__uint_as_float(v[8 + e])),
                      static_cast<double>(__uint_as_float(v[16 + e])));
    };
    // exact scales: fp64 maximum over the candidate elements (one a lane)
    double m0 = 0.0, m1 = 0.0;
    if (lane < nc * U) {
      const int ent = lane / U, e = lane % U;
      const uint32_t hd = static_cast<uint32_t>(ue[ent]);
      const int c = U * static_cast<int>(hd & 0x7FFFFFFFu) + e;
      if (c < n) {
        const double v = fabs(in64(ent, e, c));
        if ((hd >> 31) == 0) m0 = v; else m1 = v;
      }
    }
    float sc[2], r32[2];
    sc[0] = __double2float_rn(__dmul_rn(warp_max_d(m0), 1.0 / static_cast<double>(QI)));
    sc[1] = NOUT == 2 ? __double2float_rn(__dmul_rn(warp_max_d(m1), 1.0 / static_cast<double>(QI)))
                      : 0.f;
#pragma unroll
    for (int o = 0; o < 2; ++o) r32[o] = sc[o] >= 1.1754943508222875e-38f ? __frcp_rn(sc[o]) : 0.f;
    if (lane == 0) {
      p.scale[0][r] = sc[0];
      if (NOUT == 2) p.scale[1][r] = sc[1];
    }
    // near-tie codes, one element pair (one INT4 byte) a lane
    for (int q = lane; q < nt * PAIRS; q += 32) {
      const int ent = kCandCap + q / PAIRS;
      const uint32_t hd = static_cast<uint32_t>(ue[ent]);
      const int o = static_cast<int>(hd >> 31);
      const int e = 2 * (q % PAIRS);
      const int c = U * static_cast<int>(hd & 0x7FFFFFFFu) + e;
      const float so = o ? sc[1] : sc[0], ro = o ? r32[1] : r32[0];
      int q2[2] = {0, 0};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        if (so != 0.f && c + h2 < n) {
          const double v = in64(ent, e + h2, c + h2);
          q2[h2] = ro != 0.f ? code_exact(v, so, __double2float_rn(v) * ro, QI) : code_of(v, so, QI);
        }
      }
      if (INT4) {
        p.y[o][r * (n / 2) + c / 2] = static_cast<uint8_t>((q2[0] & 0xF) | ((q2[1] & 0xF) << 4));
      } else {
        p.y[o][r * n + c] = static_cast<uint8_t>(q2[0]);
        if (c + 1 < n) p.y[o][r * n + c + 1] = static_cast<uint8_t>(q2[1]);
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    h->cnt[0] = 0;
    h->cnt[1] = 0;
    h->flags = 0;
  }
}

// ---------------------------------------------------------------- exchange

// How the threads sharing a row meet: one CTA, or a cluster through
// distributed shared memory.
template <bool CL>
struct Exchange {
  cg::cluster_group cluster;
  int cl, rank;
  __device__ __forceinline__ Exchange() : cluster(cg::this_cluster()) {
    if (CL) {
      cl = static_cast<int>(cluster.num_blocks());
      rank = static_cast<int>(cluster.block_rank());
    } else {
      cl = 1;
      rank = 0;
    }
  }
  __device__ __forceinline__ void sync() {
    if (CL) cluster.sync(); else __syncthreads();
  }
  template <class V>
  __device__ __forceinline__ void publish(V *slots, int idx, V v) {  // to every CTA's copy
    if (CL) {
      for (int r = 0; r < cl; ++r) cluster.map_shared_rank(slots, r)[idx] = v;
    } else {
      slots[idx] = v;
    }
  }
  __device__ __forceinline__ void flag(int *flags, int par, int bits) {
    if (CL) {
      for (int r = 0; r < cl; ++r) atomicOr(cluster.map_shared_rank(flags, r) + par, bits);
    } else {
      atomicOr(flags + par, bits);
    }
  }
  // the row records live in the first CTA of the cluster
  __device__ __forceinline__ unsigned char *first_cta(unsigned char *q) {
    if constexpr (CL) return cluster.map_shared_rank(q, 0);
    return q;
  }
};

// ---------------------------------------------------------------- row kernel

// The row kernel's body; the __global__ entry points below differ only in
// their register budget.
template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD, bool CL>
__device__ __forceinline__ void rows_body(const KParams &p) {
  using C = Cvt<T>;
  constexpr int U = (MODE == LOAD_SCALAR) ? 2 : 8;  // elements per unit
  constexpr int W = U / 2;                          // element pairs per unit
  constexpr int QI = INT4 ? 7 : 127;
  constexpr float QF = static_cast<float>(QI);
  constexpr int NIN = ADD ? 2 : 1;                  // staged inputs per row

  // Launched as a programmatic dependent: everything before this kernel on
  // the stream is complete, and its memory visible, only from here on.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  Exchange<CL> ex;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int cl = ex.cl;
  const int rank = ex.rank;
  const int64_t cluster_id = blockIdx.x / cl;
  const int64_t nclusters = gridDim.x / cl;
  const int nslots = cl * nwarps;
  const int my_slot = rank * nwarps + warp;
  const int n = p.n;
  const int ring_depth = (MODE == LOAD_STAGED) ? p.stages : 0;  // stages in the layout
  const int stages = (MODE == LOAD_STAGED) ? p.stages : 1;      // ring arithmetic

  const int seg_begin = CL ? rank * p.seg_units : 0;  // a CTA alone holds the whole row
  const int seg_end = CL ? min(seg_begin + p.seg_units, p.units) : p.units;
  const int seg_len = max(seg_end - seg_begin, 0);
  const uint32_t seg_bytes = static_cast<uint32_t>(seg_len) * 16u;  // staged: bytes per input
  const uint32_t stage_bytes = NIN * static_cast<uint32_t>(p.seg_units) * 16u;

  extern __shared__ __align__(128) unsigned char smem[];
  // 16-byte units keep B_k in shared memory (registers go to x and G_k)
  constexpr bool BSM = (W == 4);
  const Layout lay = make_layout(nslots, NOUT, ring_depth, p.rec_bytes,
                                 bsm_bytes_for(BSM, NOUT, UPT, static_cast<int>(blockDim.x)));
  float4 *bsm = reinterpret_cast<float4 *>(smem + lay.bsm);
  auto bsm_at = [&](int o, int k, int j) -> float4 & {
    return bsm[((o * UPT + k) * 2 + j) * static_cast<int>(blockDim.x) + tid];
  };
  double *ss_slots = reinterpret_cast<double *>(smem + lay.ss);      // [nslots]
  float *wmax_slots = reinterpret_cast<float *>(smem + lay.wmax);    // [NOUT][nslots]
  float *maxb_slots = reinterpret_cast<float *>(smem + lay.maxb);    // [NOUT][nslots]
  int *rflags = reinterpret_cast<int *>(smem + lay.flags);           // [2]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars);
  int64_t *srow = reinterpret_cast<int64_t *>(smem + lay.srow);
  unsigned char *ring = smem + lay.ring;

  // ---- the first rows' copies go out before anything else (the parameter
  // loads and the set-up exchange overlap them).  The other threads wait on
  // the barriers only after the set-up exchange below.
  // staged: row `row` goes to stage s, x1 then x2; the barrier expects `hold`
  // bytes more than the copies bring (testing only: then the wait runs out)
  uint64_t policy = 0;
  auto issue = [&](int64_t row, int s, uint32_t hold) {
    const uint32_t bar = smem_addr(&bars[s]);
    const uint32_t dst = smem_addr(ring + static_cast<size_t>(s) * stage_bytes);
    const int64_t off = row * n + static_cast<int64_t>(seg_begin) * 8;
    mbar_arrive_expect_tx(bar, NIN * seg_bytes + hold);
    bulk_g2s(dst, p.x1 + off, seg_bytes, bar, policy);
    if (ADD) bulk_g2s(dst + seg_bytes, p.x2 + off, seg_bytes, bar, policy);
  };
  if (MODE == LOAD_STAGED && tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // The rows a CTA (cluster) takes, in order, as the thread that issues the
  // copies sees them: rows below p.dyn_base are dealt out in turn (c, c + G,
  // ...); the others are handed out one at a time by the workspace counter,
  // so that CTAs that run faster take more of them.  A ticket is fetched one
  // take ahead: its latency overlaps a row.  -1: no more rows.
  // The hand-out state lives in shared memory (registers are scarce), all but
  // the prefetched ticket, whose load is waited for only at the next take.
  const bool dyn = MODE == LOAD_STAGED && !CL && p.dyn_base < p.rows;
  TakeState *ts = reinterpret_cast<TakeState *>(smem + lay.take);
  int ticket = 0;
  auto take = [&]() -> int64_t {
    const int64_t nx = ts->nxt;
    if (nx < p.dyn_base) {
      ts->nxt = nx + nclusters;
      if (dyn && nx + nclusters >= p.dyn_base) ticket = atomicAdd(p.sched, 1);  // the first ticket
      return nx < p.rows ? nx : -1;
    }
    if (!dyn || ts->dry) return -1;
    const int64_t r = p.dyn_base + ticket;
    if (r >= p.rows || r < p.dyn_base) {
      ts->dry = 1;
      return -1;
    }
    ticket = atomicAdd(p.sched, 1);
    ts->ndyn += 1;
    return r;
  };
  if (MODE == LOAD_STAGED && tid == 0) {
    ts->nxt = cluster_id;
    ts->ndyn = 0;
    ts->dry = 0;
    policy = policy_evict_normal();
    for (int s = 0; s < stages; ++s) {
      const int64_t row = take();
      srow[s] = row;
      if (row >= 0 && seg_len > 0) issue(row, s, s == 0 ? p.test_hold_tx : 0u);
    }
  }

  // ---- folded parameters for this thread's units: input_k = x*rinv*G_k + B_k
  float2 G[NOUT][UPT][W], B[NOUT][UPT][W];
  float maxB[NOUT];
#pragma unroll
  for (int o = 0; o < NOUT; ++o) maxB[o] = 0.f;
#pragma unroll
  for (int k = 0; k < UPT; ++k) {
    const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
    const bool ok = u < seg_end;
    uint32_t gw[W], bw[W], sw[NOUT][W];
#pragma unroll
    for (int i = 0; i < W; ++i) {
      gw[i] = bw[i] = 0u;
#pragma unroll
      for (int o = 0; o < NOUT; ++o) sw[o][i] = 0u;
    }
    if (ok) {
      if (MODE != LOAD_SCALAR) {
        const uint4 g = ld_param16(p.gamma + static_cast<int64_t>(u) * 8);
        gw[0] = g.x; gw[1] = g.y; gw[2] = g.z; gw[3] = g.w;
        if (p.flags & F_BETA) {
          const uint4 b = ld_param16(p.beta + static_cast<int64_t>(u) * 8);
          bw[0] = b.x; bw[1] = b.y; bw[2] = b.z; bw[3] = b.w;
        }
#pragma unroll
        for (int o = 0; o < NOUT; ++o) {
          if (p.smooth[o]) {
            const uint4 s = ld_param16(p.smooth[o] + static_cast<int64_t>(u) * 8);
            sw[o][0] = s.x; sw[o][1] = s.y; sw[o][2] = s.z; sw[o][3] = s.w;
          }
        }
      } else {
        const int j = 2 * u;
        const bool two = j + 1 < n;
        gw[0] = static_cast<uint32_t>(__ldg(p.gamma + j)) |
                (two ? static_cast<uint32_t>(__ldg(p.gamma + j + 1)) << 16 : 0u);
        if (p.flags & F_BETA)
          bw[0] = static_cast<uint32_t>(__ldg(p.beta + j)) |
                  (two ? static_cast<uint32_t>(__ldg(p.beta + j + 1)) << 16 : 0u);
#pragma unroll
        for (int o = 0; o < NOUT; ++o)
          if (p.smooth[o])
            sw[o][0] = static_cast<uint32_t>(__ldg(p.smooth[o] + j)) |
                       (two ? static_cast<uint32_t>(__ldg(p.smooth[o] + j + 1)) << 16 : 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < W; ++i) {
      const float2 g2 = C::f2(gw[i]);
      const float2 b2 = C::f2(bw[i]);
#pragma unroll
      for (int o = 0; o < NOUT; ++o) {
        const float2 s2 = p.smooth[o] ? C::f2(sw[o][i]) : make_float2(1.f, 1.f);
        G[o][k][i] = __fmul2_rn(g2, s2);  // exact: two 8- (or 11-) bit significands
        B[o][k][i] = __fmul2_rn(b2, s2);
        maxB[o] = fmaxf(maxB[o], fmaxf(fabsf(B[o][k][i].x), fabsf(B[o][k][i].y)));
      }
    }
    if (BSM) {  // read back only by this thread
#pragma unroll
      for (int o = 0; o < NOUT; ++o)
#pragma unroll
        for (int j = 0; j < W / 2; ++j)
          bsm_at(o, k, j) = make_float4(B[o][k][2 * j].x, B[o][k][2 * j].y, B[o][k][2 * j + 1].x,
                                        B[o][k][2 * j + 1].y);
    }
  }
  // B_k of unit k, output o: from shared memory (16-byte units) or registers
  auto b_of = [&](int o, int k, float2 (&bk)[W]) {
#pragma unroll
    for (int i = 0; i < W; ++i) bk[i] = B[o][k][i];
    if (BSM) {
#pragma unroll
      for (int j = 0; j < W / 2; ++j) {
        const float4 b = bsm_at(o, k, j);
        bk[2 * j] = make_float2(b.x, b.y);
        bk[2 * j + 1] = make_float2(b.z, b.w);
      }
    }
  };

  // ---- set-up exchange: the row-wide bound on |B_k|; shared state; staged ring
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    const float v = warp_max_nonneg(maxB[o]);
    if (lane == 0) ex.publish(maxb_slots, o * nslots + my_slot, v);
  }
  if (tid < 2) rflags[tid] = 0;
  // the record of row iteration i: slot i % 3, in the shared memory of the
  // cluster's first CTA
  unsigned char *const recs = ex.first_cta(smem + lay.recs);
  auto slot = [&](int64_t i) -> RecHead * {
    return reinterpret_cast<RecHead *>(recs + static_cast<int>(i % 3) * p.rec_bytes);
  };
  if (rank == 0 && tid < 3) {
    RecHead *h = reinterpret_cast<RecHead *>(smem + lay.recs + tid * p.rec_bytes);
    h->cnt[0] = h->cnt[1] = 0;
    h->flags = 0;
  }
  ex.sync();
  float maxBg[NOUT];  // bound on |B_k| over the whole row
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    float m = 0.f;
    for (int i = lane; i < nslots; i += 32) m = fmaxf(m, maxb_slots[o * nslots + i]);
    maxBg[o] = warp_max_nonneg(m);
  }

  // the codes of unit u (8 or 2 elements, low bits of bits[]) of row `row`
  auto store_codes = [&](uint8_t *y, int64_t row, int u, const uint32_t (&bits)[2 * W]) {
    if (MODE != LOAD_SCALAR) {
      if (INT4) {  // 8 codes -> 4 bytes, even column in the low nibble
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= (bits[e] & 0xFu) << (4 * e);
        __stcs(reinterpret_cast<unsigned int *>(y + row * (n / 2) + static_cast<int64_t>(u) * 4),
               w);
      } else {     // 8 codes -> 8 bytes
        const uint32_t lo = __byte_perm(__byte_perm(bits[0], bits[1], 0x0040),
                                        __byte_perm(bits[2], bits[3], 0x0040), 0x5410);
        const uint32_t hi = __byte_perm(__byte_perm(bits[4], bits[5], 0x0040),
                                        __byte_perm(bits[6], bits[7], 0x0040), 0x5410);
        __stcs(reinterpret_cast<uint2 *>(y + row * n + static_cast<int64_t>(u) * 8),
               make_uint2(lo, hi));
      }
    } else {
      if (INT4) {
        y[row * (n / 2) + u] = static_cast<uint8_t>((bits[0] & 0xFu) | ((bits[1] & 0xFu) << 4));
      } else {
        const int64_t j = row * n + 2 * static_cast<int64_t>(u);
        y[j] = static_cast<uint8_t>(bits[0] & 0xFFu);
        if (2 * u + 1 < n) y[j + 1] = static_cast<uint8_t>(bits[1] & 0xFFu);
      }
    }
  };

  // ---- row records: unit u of output o on list l (0 candidate, 1 near tie) of
  // the current row, with its G_k and B_k; an overflowing list only counts,
  // and the row goes to the slow path
  int64_t it = 0;          // rows this CTA (cluster) has processed
  auto record = [&](int l, int u, int o, const float2 (&gk)[W], const float2 (&bk)[W]) {
    RecHead *h = slot(it);
    const int k = atomicAdd(&h->cnt[l], 1);
    if (k >= (l == 0 ? kCandCap : p.tie_cap)) return;
    const int ent = l == 0 ? k : kCandCap + k;
    rec_ue(h)[ent] = static_cast<int>(static_cast<uint32_t>(u) | (static_cast<uint32_t>(o) << 31));
    float *v = reinterpret_cast<float *>(rec_ent(h, p.tie_cap, ent));
    if (W == 4) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        reinterpret_cast<float4 *>(v + 8)[j] = make_float4(gk[2 * j].x, gk[2 * j].y,
                                                           gk[2 * j + 1].x, gk[2 * j + 1].y);
        reinterpret_cast<float4 *>(v + 16)[j] = make_float4(bk[2 * j].x, bk[2 * j].y,
                                                            bk[2 * j + 1].x, bk[2 * j + 1].y);
      }
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        reinterpret_cast<float2 *>(v + 8)[i] = gk[i];
        reinterpret_cast<float2 *>(v + 16)[i] = bk[i];
      }
    }
  };
  // the settling warp: the last warp of the cluster's first CTA
  const bool settler = rank == 0 && warp == nwarps - 1;

  int stage = 0;           // staged: it % stages, kept incrementally
  uint32_t phase = 0;      // staged: (it / stages) & 1, the mbarrier phase to wait for
  int64_t prev_row = -1;   // the row of the previous iteration
  int64_t prev2_row = -1;  // and of the one before
  for (;; ++it) {
    int64_t row;
    if (MODE == LOAD_STAGED) {
      row = srow[stage];
      if (row < 0) break;
    } else {
      row = cluster_id + it * nclusters;
      if (row >= p.rows) break;
    }
    const int par = static_cast<int>(it & 1);
    bool timed_out = false;
    if (MODE == LOAD_STAGED && seg_len > 0) {
      timed_out = !mbar_wait_bounded(smem_addr(&bars[stage]), phase, p.wait_limit_ns);
    }

    // ---- pass 1: x = RN16(x1 + x2) (or x1), xOut, sum of squares (fp64)
    float2 xf[UPT][W];
    double ss = 0.0;
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
      const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
      const bool ok = u < seg_end;
      uint32_t a[W], b[W];
#pragma unroll
      for (int i = 0; i < W; ++i) a[i] = b[i] = 0u;
      if (ok) {
        if (MODE == LOAD_VEC) {
          const int64_t off = row * n + static_cast<int64_t>(u) * 8;
          const uint4 va = ld_stream16(p.x1 + off);
          a[0] = va.x; a[1] = va.y; a[2] = va.z; a[3] = va.w;
          if (ADD) {
            const uint4 vb = ld_stream16(p.x2 + off);
            b[0] = vb.x; b[1] = vb.y; b[2] = vb.z; b[3] = vb.w;
          }
        } else if (MODE == LOAD_STAGED) {
          const unsigned char *st = ring + static_cast<size_t>(stage) * stage_bytes;
          const uint4 va = *reinterpret_cast<const uint4 *>(st + (u - seg_begin) * 16);
          a[0] = va.x; a[1] = va.y; a[2] = va.z; a[3] = va.w;
          if (ADD) {
            const uint4 vb =
                *reinterpret_cast<const uint4 *>(st + seg_bytes + (u - seg_begin) * 16);
            b[0] = vb.x; b[1] = vb.y; b[2] = vb.z; b[3] = vb.w;
          }
        } else {
          const int64_t j = row * n + 2 * static_cast<int64_t>(u);
          const bool two = 2 * u + 1 < n;
          a[0] = static_cast<uint32_t>(__ldcs(p.x1 + j)) |
                 (two ? static_cast<uint32_t>(__ldcs(p.x1 + j + 1)) << 16 : 0u);
          if (ADD)
            b[0] = static_cast<uint32_t>(__ldcs(p.x2 + j)) |
                   (two ? static_cast<uint32_t>(__ldcs(p.x2 + j + 1)) << 16 : 0u);
        }
      }
      uint32_t xo[W];
#pragma unroll
      for (int i = 0; i < W; ++i) {
        xo[i] = ADD ? C::add2(a[i], b[i]) : a[i];
        const float2 xv = C::f2(xo[i]);  // the x that is normalised
        xf[k][i] = xv;
        ss = __fma_rn(static_cast<double>(xv.x), static_cast<double>(xv.x), ss);
        ss = __fma_rn(static_cast<double>(xv.y), static_cast<double>(xv.y), ss);
      }
      if (ADD && ok && (p.flags & F_XOUT)) {
        if (MODE != LOAD_SCALAR) {
          *reinterpret_cast<uint4 *>(p.x_out + row * n + static_cast<int64_t>(u) * 8) =
              make_uint4(xo[0], xo[1], xo[2], xo[3]);
        } else {
          const int64_t j = row * n + 2 * static_cast<int64_t>(u);
          p.x_out[j] = static_cast<uint16_t>(xo[0] & 0xFFFFu);
          if (2 * u + 1 < n) p.x_out[j + 1] = static_cast<uint16_t>(xo[0] >> 16);
        }
      }
    }

    // ---- exchange 1: sum of squares; the previous row's flags
    {
      const double v = warp_sum_d(ss);
      const bool any_to = __any_sync(0xFFFFFFFFu, timed_out);
      if (lane == 0) {
        ex.publish(ss_slots, my_slot, v);
        if (any_to) ex.flag(rflags, par ^ 1, RF_ABORT);
      }
    }
    ex.sync();
    const int fl = rflags[par ^ 1];

    if (MODE == LOAD_STAGED) {
      if (fl & RF_ABORT) {
        // A copy never completed: record it, wait (bounded) for the copies this
        // CTA still has in flight, and stop.  Every CTA of the cluster sees the
        // flag after the same barrier.
        if (tid == 0) {
          if (atomicCAS(p.status, 0, DEV_TIMEOUT) == 0) {
            *reinterpret_cast<volatile int64_t *>(p.status + 2) = row;
          }
          if (seg_len > 0) {
            for (int s = 0; s < stages; ++s) {
              const int64_t it2 = it + s;  // the ring's outstanding iterations
              if (srow[it2 % stages] < 0) break;
              mbar_wait_bounded(smem_addr(&bars[it2 % stages]),
                                static_cast<uint32_t>((it2 / stages) & 1), p.wait_limit_ns);
            }
          }
        }
        break;
      }
      // every thread has read this stage (and its row): refill it
      if (tid == 0) {
        const int64_t nrow = take();
        srow[stage] = nrow;
        if (nrow >= 0 && seg_len > 0) issue(nrow, stage, 0u);
      }
    }

    double ss_row = 0.0;
    if (nslots <= 8) {  // every lane adds the few partial sums itself
      for (int i = 0; i < nslots; ++i) ss_row = __dadd_rn(ss_row, ss_slots[i]);
    } else {
      for (int i = lane; i < nslots; i += 32) ss_row = __dadd_rn(ss_row, ss_slots[i]);
      ss_row = warp_sum_d(ss_row);
    }
    // v = ss/n + eps; 1/sqrt(v) in binary32 for the bulk
    const double v64 = __fma_rn(ss_row, p.inv_n, static_cast<double>(p.eps));
    const float v32 = __double2float_rn(v64);
    float2 rinv2;
    {
      const float r = rsqrt_refined(v32);
      rinv2 = make_float2(r, r);
    }
    // the record: this row's sum of squares and flags (outside the normal
    // binary32 range the bulk arithmetic is not trusted: the slow path)
    if (tid == 0 && rank == 0) {
      RecHead *h = slot(it);
      h->ss = ss_row;
      h->flags = (v32 >= 1.1754943508222875e-38f && v32 <= 3.4028234663852886e+38f) ? 0 : RF_REDO;
    }

    // ---- pass 2: binary32 maxima of |input_k|, per unit and over the row
    float mu[NOUT][UPT];
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < UPT; ++k) {
        float mk = 0.f;
        float2 bk[W];
        b_of(o, k, bk);
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], bk[i]);
          if (NOUT == 1) xf[k][i] = in;  // one output: pass 3 quantizes this input
          mk = fmaxf(mk, fmaxf(fabsf(in.x), fabsf(in.y)));
        }
        mu[o][k] = mk;
        m = fmaxf(m, mk);
      }
      const float wm = warp_max_nonneg(m);
      if (lane == 0) ex.publish(wmax_slots, o * nslots + my_slot, wm);
    }
    // ---- exchange 2: row maxima
    ex.sync();
    if (tid == 0) rflags[par ^ 1] = 0;

    // ---- pass 3: quantize with the approximate scale s~ = max / Q (rounded half
    // to even via the 1.5*2^23 trick); record the candidate units and the
    // units with a code near a half-way point
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float gm = 0.f;
      for (int i = lane; i < nslots; i += 32) gm = fmaxf(gm, wmax_slots[o * nslots + i]);
      gm = warp_max_nonneg(gm);
      // s~ = gm * RN32(1/Q): within 2u of gm / Q (the error bound below allows it)
      const float sa = gm * (1.f / QF);
      const bool normal = sa >= 1.1754943508222875e-38f;
      // 1/s~ would overflow: the slow path
      if (sa != 0.f && !normal && tid == 0 && rank == 0) slot(it)->flags = RF_REDO;
      const float r32 = normal ? __frcp_rn(sa) : 0.f;
      // candidates for the row maximum: every binary32 input is within
      // 3u|input| + 12u max|B| of its value scaled by the row's common 1/Rms
      // error: the true maximum's unit is at or above thr
      const float thr = gm - 12.f * kUnit * gm - 24.f * kUnit * maxBg[o];
      // |t - t_exact| <= tau: the binary32 error of t (12u(Q + |B| r) + 2uQ) plus
      // the distance between s~ and the exact scale (10uQ + 6u maxB r)
      const float tau = 24.f * kUnit * QF + 18.f * kUnit * maxBg[o] * r32;
      const float lim = 0.5f - tau;
      const float2 r2 = make_float2(r32, r32);
      uint8_t *y = p.y[o];
#pragma unroll
      for (int k = 0; k < UPT; ++k) {
        const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
        if (u >= seg_end) continue;
        if (gm > 0.f && mu[o][k] >= thr) {  // about one unit a row
          float2 bk[W];
          b_of(o, k, bk);
          record(0, u, o, G[o][k], bk);
        }
        uint32_t bits[2 * W];  // low bits: the code (two's complement)
        float dmax = 0.f;      // largest |t - RNE(t)| of the unit
        float2 bk[W];
#pragma unroll
        for (int i = 0; i < W; ++i) bk[i] = make_float2(0.f, 0.f);
        if (NOUT == 2) b_of(o, k, bk);
#pragma unroll
        for (int i = 0; i < W; ++i) {
          // the same binary32 input as in pass 2: kept (one output) or recomputed
          const float2 in =
              NOUT == 1 ? xf[k][i] : __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], bk[i]);
          const float2 t = __fmul2_rn(in, r2);
          const float2 m = __fadd2_rn(t, make_float2(kMagic, kMagic));
          const float2 rr = __fadd2_rn(m, make_float2(-kMagic, -kMagic));  // RNE(t), exact
          const float2 d = __ffma2_rn(rr, make_float2(-1.f, -1.f), t);     // t - RNE(t), exact
          bits[2 * i] = __float_as_uint(m.x);
          bits[2 * i + 1] = __float_as_uint(m.y);
          dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        }
        store_codes(y, row, u, bits);
        // some code of the unit is near a half-way point (rare): record the unit
        if (dmax > lim) {
          if (NOUT == 1) b_of(o, k, bk);
          record(1, u, o, G[o][k], bk);
        }
      }
    }
    if (MODE == LOAD_STAGED && ++stage == stages) {
      stage = 0;
      phase ^= 1u;
    }
    // ---- the settling warp, while the next row's copy is in flight: the
    // previous row's record is complete (two barriers have passed since):
    // fetch its units' x; the row before that has its x in place: settle it
    if (settler) {
      if (it >= 1) prefetch_record<ADD, U>(p, slot(it - 1), prev_row, lane);
      if (it >= 2) {
        cp_async_wait<1>();
        __syncwarp();
        settle_record<T, INT4, NOUT, ADD, U>(p, slot(it - 2), prev2_row, lane);
      }
    }
    prev2_row = prev_row;
    prev_row = row;
  }

  // the next kernel on the stream may start its set-up (it waits for this
  // grid's completion before it reads anything)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ---- settle the last two rows (rows 0 .. it-1 are complete; all but the
  // last two are settled, and the x of row it-2 is on its way)
  if (it >= 1) {
    ex.sync();
    if (settler) {
      prefetch_record<ADD, U>(p, slot(it - 1), prev_row, lane);
      if (it >= 2) {
        cp_async_wait<1>();
        __syncwarp();
        settle_record<T, INT4, NOUT, ADD, U>(p, slot(it - 2), prev2_row, lane);
      }
      cp_async_wait<0>();
      __syncwarp();
      settle_record<T, INT4, NOUT, ADD, U>(p, slot(it - 1), prev_row, lane);
    }
  }
  // ---- the last CTA to finish returns the hand-out counters to zero (every
  // CTA's tickets are taken before it counts itself done) and checks that
  // every dynamic row was handed out exactly once and each CTA drew one empty
  // ticket: counters that were not zero when the call started fail this
  if (dyn && tid == 0) {
    atomicAdd(p.sched + 2, ts->ndyn);
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      __threadfence();
      const int handed = atomicExch(p.sched, 0);
      const int taken = atomicExch(p.sched + 2, 0);
      atomicExch(p.sched + 1, 0);
      const int64_t pool = p.rows - p.dyn_base;
      if ((static_cast<int64_t>(taken) != pool ||
           static_cast<int64_t>(handed) != pool + gridDim.x) &&
          atomicCAS(p.status, 0, DEV_SCHED) == 0)
        *reinterpret_cast<volatile int64_t *>(p.status + 2) = -1;
    }
  }
}

// At most 128 registers a thread (two 256-thread CTAs per SM), whatever the
// launch bound allows.
template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD, bool CL>
__global__ void __launch_bounds__(max_threads_for(MODE, UPT, NOUT),
                                  max_threads_for(MODE, UPT, NOUT) <= 256 ? 2 : 1)
    rows_kernel(const __grid_constant__ KParams p) {
  rows_body<T, INT4, MODE, UPT, NOUT, ADD, CL>(p);
}

// 16-byte units, four per thread, one output: at most 96 registers, so that
// five 128-thread CTAs (five rows in flight) fit an SM's 64K registers.
constexpr int kRegsUpt4 = 96;
template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD, bool CL>
__global__ void __maxnreg__(kRegsUpt4) rows_kernel_r96(const __grid_constant__ KParams p) {
  rows_body<T, INT4, MODE, UPT, NOUT, ADD, CL>(p);
}

}  // namespace arnq
