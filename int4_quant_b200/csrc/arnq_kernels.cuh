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
// A CTA (or a thread-block cluster of `cl` CTAs, for long rows or too few rows
// to fill the SMs) takes one row at a time; a thread keeps its elements of x
// and its folded parameters in registers.  Persistent grid: cluster c handles
// rows c, c + nclusters, ...  Two barriers per row: after the sum of squares,
// and after the row maximum.
//
// Arithmetic.  The bulk of the work is binary32, two lanes at a time with the
// sm_100 packed instructions (add/mul/fma.rn.f32x2):
//   x = RNE16(x1 + x2)                    -> xOut, kept as fp32 in registers
//   ss = sum x^2                          fp64 (x^2 is exact; the sum agrees with
//                                         an fp64 evaluation of the definition)
//   Rms = sqrt(ss/n + eps)                fp64, once per warp; 1/Rms also binary32
//   input_k = x*rinv*G_k + B_k            G_k = gamma*smooth_k, B_k = beta*smooth_k,
//                                         exact products of two 16-bit values
//   amax_k = max |input_k|                binary32 scan; each warp re-evaluates in
//                                         fp64 the elements within the error bound
//                                         of its own maximum (the row's true
//                                         maximum is among them), so
//   scale_k = fp32(amax_k / Q)            equals the fp64 evaluation's scale
//   t = input_k * (1/scale_k)             rounded half-to-even by adding 1.5*2^23
// |t - t_exact| <= 7u|t| + 6u|B_k|/scale_k (u = 2^-24).  A code whose binary32
// quotient lies within that bound of a half-way point is recomputed in fp64,
// ((x / Rms) * G_k + B_k) / scale_k, so every rounding decision is the one an
// fp64 evaluation of the definition makes.  Nothing here is a contraction: no
// tensor cores.
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
enum : int { DEV_TIMEOUT = 11 };

// A bounded wait gives up after this long (nanoseconds of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Shared-memory layout, sized by the launch (the host computes the same):
//   ss    [cl * nwarps] doubles: per-warp partial sums of squares of a row
//   cand  [NOUT][cl * nwarps] doubles: per-warp fp64 row maxima of |input_k|
//   maxb  [NOUT][cl * nwarps] floats: set-up reduction of the bound on |B_k|
//   abort int; bars [stages] mbarriers; ring [stages] rows of staged input
constexpr int kMaxStagesDev = 8;
struct Layout {
  int ss, cand, maxb, abort, bars, ring;
};
__host__ __device__ inline Layout make_layout(int nslots, int nout, int stages) {
  Layout L;
  int off = 0;
  L.ss = off;    off += nslots * 8;
  L.cand = off;  off += nout * nslots * 8;
  L.maxb = off;  off += nout * nslots * 4;
  off = (off + 7) & ~7;
  L.abort = off; off += 8;
  L.bars = off;  off += stages * 8;
  L.ring = (off + 127) & ~127;
  return L;
}

struct KParams {
  const uint16_t *x1, *x2, *gamma, *beta;
  const uint16_t *smooth[2];  // per output slot; nullptr = no smooth scale
  uint8_t *y[2];              // per output slot
  float *scale[2];            // per output slot
  uint16_t *x_out;
  int32_t *status;            // workspace status block (staged kernel only)
  int64_t rows;
  int32_t n;                  // row length in elements
  int32_t units;              // units per row: ceil(n / U)
  int32_t seg_units;          // units per CTA of a cluster
  int32_t flags;
  int32_t stages;             // staged kernel: ring depth
  float eps;
  double inv_n;               // 1 / n
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

// Waits for the given phase parity of an mbarrier, at most kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.  Evict-first in L2: every
// input byte is read exactly once.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
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
// Threads per CTA the register budget allows.  A thread keeps, per element, x
// and per output G and B: (1 + 2*NOUT) floats.  Up to 48 of them fit the 64
// registers of a 1024-thread CTA, up to 112 the 128 of 512 threads; more get 255.
__host__ __device__ constexpr int max_threads_for(int mode, int upt, int nout) {
  return (upt * (mode == LOAD_SCALAR ? 2 : 8) * (1 + 2 * nout) <= 48)    ? 1024
         : (upt * (mode == LOAD_SCALAR ? 2 : 8) * (1 + 2 * nout) <= 112) ? 512
                                                                         : 256;
}

constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: v + kMagic = RNE(v) + kMagic
constexpr uint32_t kMagicBits = 0x4B400000u;  // its bit pattern; low bits then hold RNE(v)
constexpr float kUnit = 5.9604644775390625e-08f;  // 2^-24, binary32 unit roundoff

// Rms(x) = sqrt(ss/n + eps) in fp64, IEEE-rounded operations in the
// definition's order.  Out of line, like the two helpers below: they run for a
// few elements per row, and inlined copies would crowd the instruction cache.
static __device__ __noinline__ double rms_exact(double ss, int n, float eps) {
  return __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(n)), static_cast<double>(eps)));
}

// |input| of one element in fp64 from the folded parameters, which are exact
// products (G = gamma*smooth, B = beta*smooth fit in binary32): |x/Rms*G + B|.
static __device__ __noinline__ double input_abs_exact(float x, float g, float b, double rms) {
  return fabs(__fma_rn(__ddiv_rn(static_cast<double>(x), rms), static_cast<double>(g),
                       static_cast<double>(b)));
}

// The code of column c decided in fp64 in the definition's order:
// round_half_even((x / Rms * gamma + beta) * smooth / scale), clamped to
// [-qmax, qmax]; returned as kMagicBits + code so its low bits pack like the
// binary32 path.  Runs only for codes within the error bound of a half-way point.
template <class T>
static __device__ __noinline__ uint32_t code_exact(const uint16_t *gamma, const uint16_t *beta,
                                                   const uint16_t *smooth, int c, float x,
                                                   double rms, float scale, int qmax) {
  int q = 0;
  if (scale != 0.f) {
    double y = __dmul_rn(__ddiv_rn(static_cast<double>(x), rms),
                         static_cast<double>(Cvt<T>::f1(__ldg(gamma + c))));
    if (beta) y = __dadd_rn(y, static_cast<double>(Cvt<T>::f1(__ldg(beta + c))));
    if (smooth) y = __dmul_rn(y, static_cast<double>(Cvt<T>::f1(__ldg(smooth + c))));
    q = __double2int_rn(__ddiv_rn(y, static_cast<double>(scale)));
    q = min(max(q, -qmax), qmax);
  }
  return kMagicBits + static_cast<uint32_t>(q);
}

// 1/sqrt(v) in binary32: the hardware estimate refined by one Newton-Raphson
// step, r' = r (3 - v r^2) / 2; within 3 ulp.
__device__ __forceinline__ float rsqrt_refined(float v) {
  const float r = rsqrtf(v);
  const float h = 0.5f * v;
  return r * __fmaf_rn(-h * r, r, 1.5f);
}

// max over lanes of non-negative floats (their bit patterns order as integers)
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v)));
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ---------------------------------------------------------------- row kernel

template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD>
__global__ void __launch_bounds__(max_threads_for(MODE, UPT, NOUT))
    rows_kernel(const KParams p) {
  using C = Cvt<T>;
  constexpr int U = (MODE == LOAD_SCALAR) ? 2 : 8;  // elements per unit
  constexpr int W = U / 2;                          // element pairs per unit
  constexpr int QI = INT4 ? 7 : 127;
  constexpr float QF = static_cast<float>(QI);
  constexpr int NIN = ADD ? 2 : 1;                  // staged inputs per row

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cluster_id = blockIdx.x / cl;
  const int64_t nclusters = gridDim.x / cl;
  const int nslots = cl * nwarps;
  const int my_slot = rank * nwarps + warp;
  const int n = p.n;
  const bool has_beta = (p.flags & F_BETA) != 0;
  const int ring_depth = (MODE == LOAD_STAGED) ? p.stages : 0;  // stages in the layout
  const int stages = (MODE == LOAD_STAGED) ? p.stages : 1;      // ring arithmetic

  const int seg_begin = rank * p.seg_units;
  const int seg_end = min(seg_begin + p.seg_units, p.units);
  const int seg_len = max(seg_end - seg_begin, 0);
  const uint32_t seg_bytes = static_cast<uint32_t>(seg_len) * 16u;  // staged: bytes per input
  const uint32_t stage_bytes = NIN * static_cast<uint32_t>(p.seg_units) * 16u;

  extern __shared__ __align__(128) unsigned char smem[];
  const Layout lay = make_layout(nslots, NOUT, ring_depth);
  double *ss_slots = reinterpret_cast<double *>(smem + lay.ss);      // [nslots]
  double *cand_slots = reinterpret_cast<double *>(smem + lay.cand);  // [NOUT][nslots]
  float *maxb_slots = reinterpret_cast<float *>(smem + lay.maxb);    // [NOUT][nslots]
  int *abort_flag = reinterpret_cast<int *>(smem + lay.abort);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars);
  unsigned char *ring = smem + lay.ring;

  auto cta_sync = [&]() {
    if (cl > 1) cluster.sync(); else __syncthreads();
  };
  // lane 0 of each warp writes one value into slot `idx` of every CTA of the cluster
  auto publish_d = [&](double *slots, int idx, double v) {
    if (cl == 1) {
      slots[idx] = v;
    } else {
      for (int r = 0; r < cl; ++r) cluster.map_shared_rank(slots, r)[idx] = v;
    }
  };

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
        if (has_beta) {
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
        if (has_beta)
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
  }

  // ---- set-up exchange: the row-wide bound on |B_k|; staged ring
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    const float v = warp_max_nonneg(maxB[o]);
    if (lane == 0) {
      if (cl == 1) {
        maxb_slots[o * nslots + warp] = v;
      } else {
        for (int r = 0; r < cl; ++r)
          cluster.map_shared_rank(maxb_slots, r)[o * nslots + my_slot] = v;
      }
    }
  }
  if (tid == 0) {
    *abort_flag = 0;
    if (MODE == LOAD_STAGED) {
      for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  cta_sync();
  float maxBg[NOUT];  // bound on |B_k| over the whole row
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    float m = 0.f;
    for (int i = lane; i < nslots; i += 32) m = fmaxf(m, maxb_slots[o * nslots + i]);
    maxBg[o] = warp_max_nonneg(m);
  }

  // staged: row `row` goes to stage s, x1 then x2
  uint64_t policy = 0;
  auto issue = [&](int64_t row, int s) {
    const uint32_t bar = smem_addr(&bars[s]);
    const uint32_t dst = smem_addr(ring + static_cast<size_t>(s) * stage_bytes);
    const int64_t off = row * n + static_cast<int64_t>(seg_begin) * 8;
    mbar_arrive_expect_tx(bar, NIN * seg_bytes);
    bulk_g2s(dst, p.x1 + off, seg_bytes, bar, policy);
    if (ADD) bulk_g2s(dst + seg_bytes, p.x2 + off, seg_bytes, bar, policy);
  };
  if (MODE == LOAD_STAGED && tid == 0 && seg_len > 0) {
    policy = policy_evict_first();
    for (int s = 0; s < stages; ++s) {
      const int64_t row = cluster_id + s * nclusters;
      if (row < p.rows) issue(row, s);
    }
  }

  int64_t it = 0;
  for (int64_t row = cluster_id; row < p.rows; row += nclusters, ++it) {
    const int stage = (MODE == LOAD_STAGED) ? static_cast<int>(it % stages) : 0;
    bool timed_out = false;
    if (MODE == LOAD_STAGED && seg_len > 0) {
      const uint32_t parity = static_cast<uint32_t>((it / stages) & 1);
      timed_out = !mbar_wait_bounded(smem_addr(&bars[stage]), parity);
    }

    // ---- pass 1: x = RNE16(x1 + x2) (or x1), xOut, sum of squares (fp64)
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
        if (ADD) {
          const float2 sum = __fadd2_rn(C::f2(a[i]), C::f2(b[i]));  // binary32 add
          xo[i] = C::pack(sum.x, sum.y);                            // RNE to 16 bits
        } else {
          xo[i] = a[i];
        }
        const float2 xv = C::f2(xo[i]);  // the x that is normalised
        xf[k][i] = xv;
        ss = __fma_rn(static_cast<double>(xv.x), static_cast<double>(xv.x), ss);
        ss = __fma_rn(static_cast<double>(xv.y), static_cast<double>(xv.y), ss);
      }
      if (ADD && ok && (p.flags & F_XOUT)) {
        if (MODE != LOAD_SCALAR) {
          __stcs(reinterpret_cast<uint4 *>(p.x_out + row * n + static_cast<int64_t>(u) * 8),
                 make_uint4(xo[0], xo[1], xo[2], xo[3]));
        } else {
          const int64_t j = row * n + 2 * static_cast<int64_t>(u);
          p.x_out[j] = static_cast<uint16_t>(xo[0] & 0xFFFFu);
          if (2 * u + 1 < n) p.x_out[j + 1] = static_cast<uint16_t>(xo[0] >> 16);
        }
      }
    }

    // ---- exchange 1: sum of squares over the row (and the abort flag)
    {
      const double v = warp_sum_d(ss);
      const bool any_to = __any_sync(0xFFFFFFFFu, timed_out);
      if (lane == 0) {
        publish_d(ss_slots, my_slot, v);
        if (any_to) {
          if (cl == 1) {
            *abort_flag = 1;
          } else {
            for (int r = 0; r < cl; ++r) *cluster.map_shared_rank(abort_flag, r) = 1;
          }
        }
      }
    }
    cta_sync();

    if (MODE == LOAD_STAGED) {
      if (*abort_flag) {
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
                                static_cast<uint32_t>((it2 / stages) & 1));
            }
          }
        }
        break;
      }
      // every thread has read this stage: refill it
      if (tid == 0 && seg_len > 0) {
        const int64_t nrow = row + static_cast<int64_t>(stages) * nclusters;
        if (nrow < p.rows) issue(nrow, stage);
      }
    }

    double ss_row = 0.0;
    for (int i = lane; i < nslots; i += 32) ss_row = __dadd_rn(ss_row, ss_slots[i]);
    ss_row = warp_sum_d(ss_row);
    // Rms in fp64 as the definition has it, computed by a lane when it first
    // needs it; 1/Rms in binary32 for the bulk
    double rms = -1.0;
    float2 rinv2;
    {
      const float v = __double2float_rn(__fma_rn(ss_row, p.inv_n, static_cast<double>(p.eps)));
      const float r = rsqrt_refined(v);
      rinv2 = make_float2(r, r);
    }

    // ---- pass 2: row maxima of |input_k|.  A binary32 scan; then every element
    // within the error bound of its warp's maximum is re-evaluated in fp64 (the
    // row's true maximum is among those of its warp) and the warp's fp64 maximum
    // is published.
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < UPT; ++k)
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
          m = fmaxf(m, fmaxf(fabsf(in.x), fabsf(in.y)));
        }
      const float wm = warp_max_nonneg(m);
      const float thr = wm - 12.f * kUnit * (wm + maxBg[o]);
      double c64 = 0.0;
      if (wm > 0.f && m >= thr) {
        if (rms < 0.0) rms = rms_exact(ss_row, n, p.eps);
#pragma unroll
        for (int k = 0; k < UPT; ++k)
#pragma unroll
          for (int i = 0; i < W; ++i) {
            const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
            if (fabsf(in.x) >= thr)
              c64 = fmax(c64, input_abs_exact(xf[k][i].x, G[o][k][i].x, B[o][k][i].x, rms));
            if (fabsf(in.y) >= thr)
              c64 = fmax(c64, input_abs_exact(xf[k][i].y, G[o][k][i].y, B[o][k][i].y, rms));
          }
      }
      c64 = warp_max_d(c64);
      if (lane == 0) publish_d(cand_slots, o * nslots + my_slot, c64);
    }
    // ---- exchange 2: fp64 row maxima
    cta_sync();

    // ---- pass 3: quantize (round half to even via the 1.5*2^23 trick) and store.
    // A zero scale gives zero codes; a scale whose reciprocal is not a normal
    // binary32 number sends every code of the row through the fp64 path.
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      double am = 0.0;
      for (int i = lane; i < nslots; i += 32) am = fmax(am, cand_slots[o * nslots + i]);
      am = warp_max_d(am);
      const float sc = __double2float_rn(__ddiv_rn(am, static_cast<double>(QI)));
      const bool tiny = sc != 0.f && sc < 1.1754943508222875e-38f;
      const float r32 = (sc == 0.f || tiny) ? 0.f : __frcp_rn(sc);
      // |t - t_exact| <= tau for the codes of this thread
      const float tau = 12.f * kUnit * (QF + maxB[o] * r32) + 2.f * kUnit * QF;
      const float lim = tiny ? -1.f : 0.5f - tau;
      if (tid == 0 && rank == 0) p.scale[o][row] = sc;
      const float2 r2 = make_float2(r32, r32);
      uint8_t *y = p.y[o];
#pragma unroll
      for (int k = 0; k < UPT; ++k) {
        const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
        if (u >= seg_end) continue;
        uint32_t bits[2 * W];  // low bits: the code (two's complement)
        float dmax = 0.f;      // largest |t - RNE(t)| of the unit
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
          const float2 t = __fmul2_rn(in, r2);
          const float2 m = __fadd2_rn(t, make_float2(kMagic, kMagic));
          const float2 rr = __fadd2_rn(m, make_float2(-kMagic, -kMagic));  // RNE(t), exact
          const float2 d = __ffma2_rn(rr, make_float2(-1.f, -1.f), t);     // t - RNE(t), exact
          bits[2 * i] = __float_as_uint(m.x);
          bits[2 * i + 1] = __float_as_uint(m.y);
          dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        }
        if (dmax > lim) {  // some code of the unit is near a half-way point (rare)
          if (rms < 0.0) rms = rms_exact(ss_row, n, p.eps);
          const uint16_t *beta = has_beta ? p.beta : nullptr;
#pragma unroll
          for (int i = 0; i < W; ++i) {
            const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
            const float2 t = __fmul2_rn(in, r2);
            const int c = U * u + 2 * i;  // column of the pair's first element
            if (fabsf(t.x - rintf(t.x)) > lim)
              bits[2 * i] = code_exact<T>(p.gamma, beta, p.smooth[o], c, xf[k][i].x, rms, sc, QI);
            if (fabsf(t.y - rintf(t.y)) > lim && c + 1 < n)
              bits[2 * i + 1] =
                  code_exact<T>(p.gamma, beta, p.smooth[o], c + 1, xf[k][i].y, rms, sc, QI);
          }
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
      }
    }
  }
  // no CTA leaves while a peer may still touch its shared memory
  if (cl > 1) cluster.sync();
}

}  // namespace arnq
