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
// A CTA (or, for rows too long for one CTA, a thread-block cluster of CTAs
// sharing a row through distributed shared memory) takes one row at a time; each thread keeps its elements of x and its folded
// parameters G_k in registers (B_k of 16-byte units in shared memory, read
// back by the thread that wrote it).  Persistent grid: a CTA (cluster) takes
// rows c, c + G, ...  Two barriers per row: after the sum of squares and
// after the row maximum.  The kernel is launched as a programmatic dependent
// (it waits for the preceding work before touching memory, or, when the
// caller promises constant parameters, before touching anything but them;
// and it lets the next kernel start its set-up after its last row).
//
// Arithmetic of the fast path, binary32 two lanes at a time with the sm_100
// packed instructions (add/mul/fma.rn.f32x2):
//   x = RN16(x1 + x2)            add.rn.{bf16,f16}x2 -- the correctly rounded
//                                sum, which equals rounding the binary32 sum
//   ss = sum x^2                 fp64 (each x^2 is exact)
//   1/Rms                        binary32 from ss (within a few ulp)
//   input_k = x*rinv*G_k + B_k   G_k = gamma*smooth_k, B_k = beta*smooth_k, exact
//                                products of two 16-bit values
//   s~_k = max|input_k| / Q      approximate scale
//   code = RNE(input_k / s~_k)   rounded half-to-even by adding 1.5*2^23
// The result must be what an fp64 evaluation of the definition gives, with the
// scale rounded to binary32: scale_k = RN32(max|input_k| / Q) and
// code = RNE(input_k / scale_k).  The fast path writes its codes and, for
// each row, a record of the few units it cannot settle (candidates for the
// row maximum, codes near a half-way point; see the records below).  After
// its last row the CTA (the cluster's first CTA) settles its rows from the
// records: the exact scale RN32(max fp64 |input| over the candidates / Q),
// then the near-tie codes, decided exactly from fp64 inputs (code_exact).
// The records hold unit indices only; the settling reads those units' x back
// from xOut (or the inputs) and the parameters from memory.  The fp64 inputs
// use 1/Rms from Newton steps (a few fp64 ulp): the decisions they settle sit
// many orders of magnitude above fp64 rounding.  A row whose record overflows
// (many equal maxima, many exact ties) or whose sum of squares or scale leaves
// the normal binary32 range is recomputed whole by its lanes, in fp64 with
// IEEE divisions in the definition's order.
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
  F_XOUT = 2,   // xOut written
  F_EARLY = 4   // parameters read before the wait for the preceding work
};
enum : int { LOAD_VEC = 0, LOAD_SCALAR = 1, LOAD_STAGED = 2 };

// status codes the kernels record in the workspace status block
enum : int {
  DEV_TIMEOUT = 11    // a bounded wait ran out
};

// A bounded wait gives up after this long (nanoseconds of %globaltimer)
// unless the launch asks for another limit.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// row flags exchanged at the first barrier of the next row
enum : int { RF_REDO = 1, RF_ABORT = 2 };

// The workspace holds only the status block (kStatusBytes; the status code
// and a row at bytes 0-15, the rest reserved).
constexpr int kStatusBytes = 256;

// Row records.  The binary32 fast path leaves a few units (8 or 2 elements)
// per row that it cannot settle: candidate units, holding an element within
// the binary32 error bound of the row maximum (the true maximum is among
// them), and near-tie units, holding a code whose binary32 quotient t lies
// within tau of a half-way point (|t - t_exact| <= tau covers the binary32
// error and the distance between s~ and the exact scale).  Each CTA (each
// cluster: in its first CTA) keeps one record per row it processes in its
// shared memory and settles them all after its last row, reading x back from
// xOut (or the inputs) and the parameters from memory.  Record:
//   header (32 B): double ss; int cnt[2] (candidate, near-tie units); int flags;
//       int pad; int64 row
//   ue [cap] ints: unit | output << 31, candidates first (cap = kCandCap + tie_cap)
// (a record holds indices only: the records of a CTA's rows share the SM's
// shared memory with the staging ring and B_k, and larger ones cost CTAs)
// A near tie needs |t - RNE(t)| > 0.5 - tau, about 2 tau ~ 1e-3 of the codes
// or fewer; tie_cap leaves several times that for a row of n columns and nout
// outputs, so rows overflow (and go to the slow path) only by design: many
// exact ties.
constexpr int kCandCap = 4;     // candidate units per row
__host__ __device__ inline int tie_cap(int n, int nout) { return 12 + (n * nout + 255) / 256; }
struct TailHead {
  double ss;
  int cnt[2];
  int flags;
  int pad;
  int64_t row;
};
// bytes of one record (a multiple of 16: the header's double stays aligned)
__host__ __device__ inline int tail_rec_bytes(int tcap) {
  return static_cast<int>(sizeof(TailHead)) + (((kCandCap + tcap) * 4 + 15) & ~15);
}

// Shared-memory layout, sized by the launch (the host computes the same):
//   ss    [nslots] doubles: per-warp partial sums
//   wmax  [NOUT][nslots] floats: per-warp binary32 row maxima of |input_k|
//   maxb  [NOUT][nslots] floats: set-up reduction of the bound on |B_k|
//   flags [2] ints: RF_* of a row, by row parity
//   bars  [stages] mbarriers
//   trec  [tail_rows] row records of trec_bytes each (used in the cluster's first CTA)
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
  int ss, wmax, maxb, flags, bars, trec, bsm, ring;
};
__host__ __device__ inline Layout make_layout(int nslots, int nout, int stages, int tail_rows,
                                              int trec_bytes, int bsm_bytes) {
  Layout L;
  int off = 0;
  L.ss = off;    off += nslots * 8;
  L.wmax = off;  off += nout * nslots * 4;
  L.maxb = off;  off += nout * nslots * 4;
  off = (off + 7) & ~7;
  L.flags = off; off += 2 * 4;
  off = (off + 7) & ~7;
  L.bars = off;  off += stages * 8;
  off = (off + 15) & ~15;
  L.trec = off;  off += tail_rows * trec_bytes;
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
  int32_t tie_cap;            // near-tie units a record holds
  int64_t rows;
  int32_t n;                  // row length in elements
  int32_t units;              // units per row: ceil(n / U)
  int32_t seg_units;          // units per CTA of a cluster
  int32_t flags;
  int32_t stages;             // staged kernel: ring depth
  int32_t tail_rows;          // records per CTA (cluster): rows it processes, at most
  int32_t trec_bytes;         // bytes per record (tail_rec_bytes)
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
// sum / max over an aligned group of `width` lanes (a power of two up to 32;
// mask: the group's lanes)
__device__ __forceinline__ double group_sum_d(double v, unsigned mask, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(mask, v, o, width));
  return v;
}
__device__ __forceinline__ double group_max_d(double v, unsigned mask, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(mask, v, o, width));
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

// round_half_even(input / scale) clamped to [-qmax, qmax]; 0 for a zero scale
__device__ __forceinline__ int code_of(double in, float scale, int qmax) {
  if (scale == 0.f) return 0;
  return code_of_t(__ddiv_rn(in, static_cast<double>(scale)), qmax);
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

// Whole row in fp64, in the definition's order, by an aligned group of
// `width` lanes (lane = 0 .. width-1, mask: the group's lanes), x read back
// from memory: the slow path for rows the fast path cannot settle.
template <class T, bool INT4, int NOUT, bool ADD>
__device__ __forceinline__ void exact_row_lanes(const KParams &p, int64_t row, int lane, int width,
                                                unsigned mask) {
  constexpr int QI = INT4 ? 7 : 127;
  const int n = p.n;
  const int64_t base = row * n;
  double ss = 0.0;
  for (int c = lane; c < n; c += width) {
    const double a = x_reload<T, ADD>(p, row, c);
    ss = __fma_rn(a, a, ss);
  }
  const double rms = rms_of(group_sum_d(ss, mask, width), n, p.eps);
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    double m = 0.0;
    for (int c = lane; c < n; c += width)
      m = fmax(m, fabs(input_of<T>(p, o, c, x_reload<T, ADD>(p, row, c), rms)));
    const float sc =
        __double2float_rn(__ddiv_rn(group_max_d(m, mask, width), static_cast<double>(QI)));
    if (lane == 0) p.scale[o][row] = sc;
    for (int c = 2 * lane; c < n; c += 2 * width) {  // element pairs: an INT4 byte has one writer
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

// ---------------------------------------------------------------- in-kernel settling

// Settles one row from its record with an aligned group of g lanes (lane l of
// g >= 8, gmask: the group's lanes): the exact scales from the candidate
// units, then the near-tie units' codes, in fp64 from x read back from memory
// and the parameters.  The loads of the
// common case (every candidate element, and each lane's first two element
// pairs of near-tie units) are issued before any arithmetic.
template <class T, bool INT4, int NOUT, bool ADD, int U>
__device__ __forceinline__ void settle_row_group(const KParams &p, int64_t r, double ss, int nc,
                                                 int nt, const int *ent, int l, int g,
                                                 unsigned gmask) {
  using C = Cvt<T>;
  constexpr int QI = INT4 ? 7 : 127;
  constexpr int PAIRS = U / 2;           // element pairs per unit
  constexpr int CE = kCandCap * U / 8;   // candidate elements per lane, at most (g >= 8)
  const int n = p.n;
  struct Elem { float x, g, b; };
  const Elem zero = {0.f, 0.f, 0.f};
  auto load = [&](int q, int o, int c) -> Elem {
    (void)q;
    Elem e;
    e.x = x_reload<T, ADD>(p, r, c);
    const float sm = p.smooth[o] ? C::f1(__ldg(p.smooth[o] + c)) : 1.f;
    e.g = C::f1(__ldg(p.gamma + c)) * sm;  // exact: two 16-bit significands
    e.b = (p.flags & F_BETA) ? C::f1(__ldg(p.beta + c)) * sm : 0.f;
    return e;
  };
  auto unit_of = [](uint32_t hd) { return static_cast<int>(hd & 0x7FFFFFFFu); };
  auto out_of = [](uint32_t hd) { return static_cast<int>(hd >> 31); };

  // candidate elements e = l, l + g, ... of the nc * U
  Elem ce[CE];
  int co[CE];
  bool cv[CE];
#pragma unroll
  for (int k = 0; k < CE; ++k) {
    const int e = l + k * g;
    ce[k] = zero;
    co[k] = 0;
    cv[k] = false;
    if (e < nc * U) {
      const uint32_t hd = static_cast<uint32_t>(ent[e / U]);
      const int c = U * unit_of(hd) + e % U;
      if (c < n) {
        co[k] = out_of(hd);
        cv[k] = true;
        ce[k] = load(e / U, co[k], c);
      }
    }
  }
  // near-tie element pairs q = l, l + g, ...: the first two now
  Elem ta[2], tb[2];
  uint32_t th[2];
  int tc[2];
  bool tv[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int q = l + k * g;
    ta[k] = tb[k] = zero;
    th[k] = 0u;
    tc[k] = 0;
    tv[k] = q < nt * PAIRS;
    if (tv[k]) {
      th[k] = static_cast<uint32_t>(ent[kCandCap + q / PAIRS]);
      tc[k] = U * unit_of(th[k]) + 2 * (q % PAIRS);
      tv[k] = tc[k] < n;  // (always: a unit of the row)
    }
    if (tv[k]) {
      ta[k] = load(kCandCap + q / PAIRS, out_of(th[k]), tc[k]);
      if (tc[k] + 1 < n) tb[k] = load(kCandCap + q / PAIRS, out_of(th[k]), tc[k] + 1);
    }
  }

  const double ri = rsqrt64(__fma_rn(ss, p.inv_n, static_cast<double>(p.eps)));
  auto input64 = [&](const Elem &e) -> double {
    return __fma_rn(__dmul_rn(static_cast<double>(e.x), ri), static_cast<double>(e.g),
                    static_cast<double>(e.b));
  };
  // exact scales: fp64 maximum over the candidate elements
  double m0 = 0.0, m1 = 0.0;
#pragma unroll
  for (int k = 0; k < CE; ++k) {
    if (cv[k]) {
      const double v = fabs(input64(ce[k]));
      if (co[k] == 0) m0 = fmax(m0, v); else m1 = fmax(m1, v);
    }
  }
  const double inv_q = 1.0 / static_cast<double>(QI);
  float sc[2] = {0.f, 0.f};
  sc[0] = __double2float_rn(__dmul_rn(group_max_d(m0, gmask, g), inv_q));
  if (NOUT == 2) sc[1] = __double2float_rn(__dmul_rn(group_max_d(m1, gmask, g), inv_q));
  if (l == 0) {
    p.scale[0][r] = sc[0];
    if (NOUT == 2) p.scale[1][r] = sc[1];
  }
  // near-tie codes in fp64, one element pair (one INT4 byte) at a time
  auto put = [&](uint32_t hd, int c, const Elem &e0, const Elem &e1) {
    const int o = out_of(hd);
    const float so = o == 0 ? sc[0] : sc[1];
    // exact decisions: code_exact with the binary32 quotient as its guide
    // (a normal scale), else an IEEE division
    auto code = [&](const Elem &el) -> int {
      const double v = input64(el);
      if (so >= 1.1754943508222875e-38f) return code_exact(v, so, __double2float_rn(v) * __frcp_rn(so), QI);
      return code_of(v, so, QI);
    };
    const int q0 = so == 0.f ? 0 : code(e0);
    const int q1 = (so == 0.f || c + 1 >= n) ? 0 : code(e1);
    if (INT4) {
      p.y[o][r * (n / 2) + c / 2] = static_cast<uint8_t>((q0 & 0xF) | ((q1 & 0xF) << 4));
    } else {
      p.y[o][r * n + c] = static_cast<uint8_t>(q0);
      if (c + 1 < n) p.y[o][r * n + c + 1] = static_cast<uint8_t>(q1);
    }
  };
#pragma unroll
  for (int k = 0; k < 2; ++k)
    if (tv[k]) put(th[k], tc[k], ta[k], tb[k]);
  for (int q = l + 2 * g; q < nt * PAIRS; q += g) {  // more than two pairs per lane
    const uint32_t hd = static_cast<uint32_t>(ent[kCandCap + q / PAIRS]);
    const int c = U * unit_of(hd) + 2 * (q % PAIRS);
    if (c >= n) continue;  // (always in the row)
    const Elem e0 = load(kCandCap + q / PAIRS, out_of(hd), c);
    const Elem e1 = c + 1 < n ? load(kCandCap + q / PAIRS, out_of(hd), c + 1) : zero;
    put(hd, c, e0, e1);
  }
}

// The CTA (the first CTA of a cluster) settles its rows (records 0 ..
// nrows-1, each naming its row) from the records in its shared memory, after
// its last row: a group of lanes per row (32, 16 or 8: as many rows at once as
// the CTA's threads allow).  Rows whose record overflowed, or that the fast
// path flagged, are recomputed whole in fp64 by their group.
template <class T, bool INT4, int NOUT, bool ADD, int U>
__device__ __forceinline__ void tail_settle(const KParams &p, const unsigned char *trec, int nrows) {
  const int nthreads = static_cast<int>(blockDim.x);
  int g = 32;
  while (g > 8 && nthreads / g < nrows) g >>= 1;
  const int groups = nthreads / g;
  const int wl = static_cast<int>(threadIdx.x) & 31;
  const int l = wl & (g - 1);
  const unsigned gmask = g == 32 ? 0xFFFFFFFFu : ((1u << g) - 1u) << (wl & ~(g - 1));
  for (int i = static_cast<int>(threadIdx.x) / g; i < nrows; i += groups) {
    const TailHead *h = reinterpret_cast<const TailHead *>(trec + static_cast<size_t>(i) * p.trec_bytes);
    const int *ent = reinterpret_cast<const int *>(h + 1);
    const int64_t r = h->row;
    const int nc = h->cnt[0], nt = h->cnt[1];
    if ((h->flags & RF_REDO) || nc > kCandCap || nt > p.tie_cap)
      exact_row_lanes<T, INT4, NOUT, ADD>(p, r, l, g, gmask);
    else
      settle_row_group<T, INT4, NOUT, ADD, U>(p, r, h->ss, nc, nt, ent, l, g, gmask);
  }
}

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
  // the stream is complete, and its memory visible, only after
  // griddepcontrol.wait.  Normally that is the first thing the kernel does.
  // With F_EARLY (the caller's promise that the preceding work does not write
  // gamma, beta or the smooth scales) the parameter loads and the set-up
  // exchange come first, overlapping the preceding work's end, and the wait
  // comes right before the first row's copies.
  const bool early = (p.flags & F_EARLY) != 0;
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
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
  const Layout lay = make_layout(nslots, NOUT, ring_depth, p.tail_rows, p.trec_bytes,
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
  unsigned char *ring = smem + lay.ring;

  // ---- the first rows' copies go out before anything else (the parameter
  // loads and the set-up exchange overlap them), unless the parameters were
  // read before the wait (then right after it).  The other threads wait on
  // the barriers only after the set-up exchange below.
  // staged: row `row` goes to stage s, x1 then x2; the barrier expects `hold`
  // bytes more than the copies bring (testing only: then the wait runs out)
  auto issue = [&](int64_t row, int s, uint32_t hold) {
    const uint64_t policy = policy_evict_normal();
    const uint32_t bar = smem_addr(&bars[s]);
    const uint32_t dst = smem_addr(ring + static_cast<size_t>(s) * stage_bytes);
    const int64_t off = row * n + static_cast<int64_t>(seg_begin) * 8;
    mbar_arrive_expect_tx(bar, NIN * seg_bytes + hold);
    bulk_g2s(dst, p.x1 + off, seg_bytes, bar, policy);
    if (ADD) bulk_g2s(dst + seg_bytes, p.x2 + off, seg_bytes, bar, policy);
  };
  auto first_copies = [&]() {
    for (int s = 0; s < stages; ++s) {
      const int64_t row = cluster_id + s * nclusters;
      if (row < p.rows && seg_len > 0) issue(row, s, s == 0 ? p.test_hold_tx : 0u);
    }
  };
  if (MODE == LOAD_STAGED && tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!early) first_copies();
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
  // the records: one per row this CTA (cluster) processes, in the shared
  // memory of the cluster's first CTA
  unsigned char *const trec = ex.first_cta(smem + lay.trec);
  auto thead = [&](int64_t i) -> TailHead * {
    return reinterpret_cast<TailHead *>(trec + static_cast<size_t>(i) * p.trec_bytes);
  };
  if (rank == 0) {
    for (int i = tid; i < p.tail_rows; i += blockDim.x) {
      TailHead *th = reinterpret_cast<TailHead *>(smem + lay.trec +
                                                  static_cast<size_t>(i) * p.trec_bytes);
      th->cnt[0] = th->cnt[1] = 0;
      th->flags = 0;
    }
  }
  ex.sync();
  if (early) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (MODE == LOAD_STAGED && tid == 0) first_copies();
  }
  float maxBg[NOUT];  // bound on |B_k| over the whole row
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    float m = 0.f;
    for (int i = lane; i < nslots; i += 32) m = fmaxf(m, maxb_slots[o * nslots + i]);
    maxBg[o] = warp_max_nonneg(m);
  }

  // ---- row records: record unit u of output o on list l (0 candidate, 1
  // near tie) of the current row; an overflowing list only counts, and the
  // row goes to the slow path.
  int64_t it = 0;          // rows this CTA (cluster) has processed
  auto record = [&](int l, int u, int o) {
    TailHead *th = thead(it);
    const int k = atomicAdd(&th->cnt[l], 1);
    if (k < (l == 0 ? kCandCap : p.tie_cap))
      reinterpret_cast<int *>(th + 1)[l == 0 ? k : kCandCap + k] =
          static_cast<int>(static_cast<uint32_t>(u) | (static_cast<uint32_t>(o) << 31));
  };
  int stage = 0;          // staged: it % stages, kept incrementally
  uint32_t phase = 0;     // staged: (it / stages) & 1, the mbarrier phase to wait for
  for (int64_t row = cluster_id; row < p.rows; row += nclusters, ++it) {
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
              if (cluster_id + it2 * nclusters >= p.rows) break;
              mbar_wait_bounded(smem_addr(&bars[it2 % stages]),
                                static_cast<uint32_t>((it2 / stages) & 1), p.wait_limit_ns);
            }
          }
        }
        break;
      }
      // every thread has read this stage: refill it
      if (tid == 0 && seg_len > 0) {
        const int64_t nrow = row + static_cast<int64_t>(stages) * nclusters;
        if (nrow < p.rows) issue(nrow, stage, 0u);
      }
    }

    double ss_row = 0.0;
    if (nslots <= 8) {  // every lane adds the few partial sums itself
      for (int i = 0; i < nslots; ++i) ss_row = __dadd_rn(ss_row, ss_slots[i]);
    } else {
      for (int i = lane; i < nslots; i += 32) ss_row = __dadd_rn(ss_row, ss_slots[i]);
      ss_row = warp_sum_d(ss_row);
    }
    // v = ss/n + eps; 1/sqrt(v) in binary32 for the bulk, in fp64 when needed
    const double v64 = __fma_rn(ss_row, p.inv_n, static_cast<double>(p.eps));
    const float v32 = __double2float_rn(v64);
    float2 rinv2;
    {
      const float r = rsqrt_refined(v32);
      rinv2 = make_float2(r, r);
    }
    // the record: this row, its sum of squares and flags (outside the normal
    // binary32 range the bulk arithmetic is not trusted)
    if (tid == 0 && rank == 0) {
      TailHead *th = thead(it);
      th->row = row;
      th->ss = ss_row;
      th->flags = (v32 >= 1.1754943508222875e-38f && v32 <= 3.4028234663852886e+38f) ? 0 : RF_REDO;
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
    // to even via the 1.5*2^23 trick); queue the codes near a half-way point
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float gm = 0.f;
      for (int i = lane; i < nslots; i += 32) gm = fmaxf(gm, wmax_slots[o * nslots + i]);
      gm = warp_max_nonneg(gm);
      // s~ = gm * RN32(1/Q): within 2u of gm / Q (the error bound below allows it)
      const float sa = gm * (1.f / QF);
      const bool normal = sa >= 1.1754943508222875e-38f;
      // 1/s~ would overflow: the slow path
      if (sa != 0.f && !normal && tid == 0 && rank == 0) {
        thead(it)->flags = RF_REDO;
      }
      const float r32 = normal ? __frcp_rn(sa) : 0.f;
      // candidates for the row maximum: within the binary32 error of it
      const float thr = gm - 12.f * kUnit * (gm + maxBg[o]);
      if (gm > 0.f) {  // about one unit per row
#pragma unroll
        for (int k = 0; k < UPT; ++k) {
          const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
          if (mu[o][k] >= thr && u < seg_end) record(0, u, o);
        }
      }
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
        if (MODE != LOAD_SCALAR) {
          if (INT4) {  // 8 codes -> 4 bytes, even column in the low nibble
            uint32_t w = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) w |= (bits[e] & 0xFu) << (4 * e);
            __stcs(reinterpret_cast<unsigned int *>(y + row * (n / 2) +
                                                    static_cast<int64_t>(u) * 4), w);
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
            y[row * (n / 2) + u] =
                static_cast<uint8_t>((bits[0] & 0xFu) | ((bits[1] & 0xFu) << 4));
          } else {
            const int64_t j = row * n + 2 * static_cast<int64_t>(u);
            y[j] = static_cast<uint8_t>(bits[0] & 0xFFu);
            if (2 * u + 1 < n) y[j + 1] = static_cast<uint8_t>(bits[1] & 0xFFu);
          }
        }
        // some code of the unit is near a half-way point (rare): record the unit
        if (dmax > lim) record(1, u, o);
      }
    }
    if (MODE == LOAD_STAGED && ++stage == stages) {
      stage = 0;
      phase ^= 1u;
    }
  }

  // the next kernel on the stream may start its set-up (it waits for this
  // grid's completion before it reads anything)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ---- settle this CTA's (cluster's) rows from their records, once the last
  // row's record is complete.  After the barrier no CTA touches a peer's
  // shared memory.
  if (it >= 1) {
    ex.sync();
    if (rank == 0) tail_settle<T, INT4, NOUT, ADD, U>(p, smem + lay.trec, static_cast<int>(it));
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
