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
// A row is split over a thread-block cluster of `cl` CTAs when it is long or
// when there are too few rows to fill the SMs; partial sums and maxima are then
// exchanged through distributed shared memory.  Persistent grid: cluster c
// handles rows c, c + nclusters, ...
//
// Arithmetic.  The bulk of the work is binary32, two lanes at a time with the
// sm_100 packed instructions (add/mul/fma.rn.f32x2):
//   x = RNE16(x1 + x2)                    -> xOut, kept as fp32 in registers
//   ss = sum x^2                          fp64 (x^2 is exact; the sum agrees with
//                                         an fp64 evaluation of the definition)
//   rinv = 1/sqrt(ss/n + eps)             fp64 per row, rounded once to fp32
//   input_k = x*rinv*G_k + B_k            G_k = gamma*smooth_k, B_k = beta*smooth_k
//   amax_k = max |input_k|                fp32 to find candidates; the candidates
//                                         are re-evaluated in fp64, so
//   scale_k = fp32(amax_k / Q)            matches an fp64 evaluation bit for bit
//   t = input_k * (1/scale_k)             rounded half-to-even by adding 1.5*2^23
// A code whose binary32 quotient t lies within the proven error bound tau of a
// half-way point is recomputed in fp64 in the definition's order
// (x / Rms * gamma + beta) * smooth / scale, so every rounding decision is the
// one an fp64 evaluation of the definition makes.  Nothing here is a
// contraction: no tensor cores.
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

// Shared-memory header: per-warp slots for the two row reductions (fp64, up to
// 16 CTAs x 32 warps, two outputs), an abort flag, up to 16 mbarriers.
constexpr int kMaxStagesDev = 16;
constexpr int kSlotsSS = 0;                        // 512 doubles
constexpr int kSlotsMax = kSlotsSS + 512 * 8;      // 512 x 2 doubles
constexpr int kAbortOff = kSlotsMax + 512 * 16;    // int
constexpr int kBarsOff = kAbortOff + 128;          // 16 x uint64
constexpr int kRingOff = kBarsOff + 8 * kMaxStagesDev;
static_assert(kRingOff % 128 == 0, "ring must stay 128-byte aligned");

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

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
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
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Threads per CTA the register budget allows: a thread keeps x (fp32) and the
// folded parameters (fp32) of its elements for every output across rows.
template <int MODE, int UPT, int NOUT>
struct MaxThreads {
  static constexpr int elems = UPT * (MODE == LOAD_SCALAR ? 2 : 8);
  static constexpr int value = (elems <= 8) ? (NOUT == 1 ? 1024 : 768) : 512;
};

constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: v + kMagic = RNE(v) + kMagic
constexpr uint32_t kMagicBits = 0x4B400000u;  // its bit pattern; low bits then hold RNE(v)
constexpr float kUnit = 5.9604644775390625e-08f;  // 2^-24, binary32 unit roundoff

// ---------------------------------------------------------------- row kernel

template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD>
__global__ void __launch_bounds__(MaxThreads<MODE, UPT, NOUT>::value)
    rows_kernel(const KParams p) {
  using C = Cvt<T>;
  constexpr int U = (MODE == LOAD_SCALAR) ? 2 : 8;  // elements per unit
  constexpr int W = U / 2;                          // element pairs per unit
  constexpr int QI = INT4 ? 7 : 127;
  constexpr float QF = static_cast<float>(QI);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cluster_id = blockIdx.x / cl;
  const int64_t nclusters = gridDim.x / cl;
  const int n = p.n;
  const bool has_beta = (p.flags & F_BETA) != 0;

  extern __shared__ __align__(128) unsigned char smem[];
  double *ss_slots = reinterpret_cast<double *>(smem + kSlotsSS);    // [cl * nwarps]
  double *max_slots = reinterpret_cast<double *>(smem + kSlotsMax);  // [NOUT][cl * nwarps]
  int *abort_any = reinterpret_cast<int *>(smem + kAbortOff);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarsOff);
  unsigned char *ring = smem + kRingOff;

  const int seg_begin = rank * p.seg_units;
  const int seg_end = min(seg_begin + p.seg_units, p.units);
  const int seg_len = max(seg_end - seg_begin, 0);
  const uint32_t seg_bytes = static_cast<uint32_t>(seg_len) * 16u;  // staged: bytes per input
  const int nslots = cl * nwarps;

  // column of element h (0/1) of pair i of this thread's k-th unit
  auto col = [&](int k, int i, int h) -> int {
    const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
    return u * U + 2 * i + h;
  };

  // ---- folded parameters for this thread's units: input_k = a * G_k + B_k
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
        auto pair = [&](const uint16_t *a) -> uint32_t {
          const uint32_t lo = __ldg(a + j);
          const uint32_t hi = two ? __ldg(a + j + 1) : 0u;
          return lo | (hi << 16);
        };
        gw[0] = pair(p.gamma);
        if (has_beta) bw[0] = pair(p.beta);
#pragma unroll
        for (int o = 0; o < NOUT; ++o)
          if (p.smooth[o]) sw[o][0] = pair(p.smooth[o]);
      }
    }
#pragma unroll
    for (int i = 0; i < W; ++i) {
      const float2 g2 = C::f2(gw[i]);
      const float2 b2 = C::f2(bw[i]);
#pragma unroll
      for (int o = 0; o < NOUT; ++o) {
        const float2 s2 = p.smooth[o] ? C::f2(sw[o][i]) : make_float2(1.f, 1.f);
        G[o][k][i] = __fmul2_rn(g2, s2);
        B[o][k][i] = __fmul2_rn(b2, s2);
        maxB[o] = fmaxf(maxB[o], fmaxf(fabsf(B[o][k][i].x), fabsf(B[o][k][i].y)));
      }
    }
  }

  // ---- staged ring set-up
  uint64_t policy = 0;
  const int stages = (MODE == LOAD_STAGED) ? p.stages : 1;
  const uint32_t stage_stride = ADD ? 2u * seg_bytes : seg_bytes;
  if (tid == 0) {
    *abort_any = 0;
    if (MODE == LOAD_STAGED) {
      for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  if (cl > 1) cluster.sync(); else __syncthreads();

  auto issue = [&](int64_t row, int s) {
    const uint32_t bar = smem_addr(&bars[s]);
    const uint32_t dst = smem_addr(ring + static_cast<size_t>(s) * stage_stride);
    const int64_t off = row * n + static_cast<int64_t>(seg_begin) * 8;
    mbar_arrive_expect_tx(bar, stage_stride);
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

  // fp64 re-evaluation of input_k at one column, in the definition's order:
  // (x / Rms * gamma + beta) * smooth_k, with Rms = sqrt(ss/n + eps).
  auto input64 = [&](int o, int c, float x, double rms) -> double {
    double y = __dmul_rn(__ddiv_rn(static_cast<double>(x), rms),
                         static_cast<double>(C::f1(p.gamma[c])));
    if (has_beta) y = __dadd_rn(y, static_cast<double>(C::f1(p.beta[c])));
    if (p.smooth[o]) y = __dmul_rn(y, static_cast<double>(C::f1(p.smooth[o][c])));
    return y;
  };

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
          const unsigned char *st = ring + static_cast<size_t>(stage) * stage_stride;
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
          const float2 s = __fadd2_rn(C::f2(a[i]), C::f2(b[i]));  // binary32 add
          xo[i] = C::pack(s.x, s.y);                              // RNE to 16 bits
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
        if (cl == 1) {
          ss_slots[warp] = v;
          if (any_to) *abort_any = 1;
        } else {
          for (int r = 0; r < cl; ++r) {
            cluster.map_shared_rank(ss_slots, r)[rank * nwarps + warp] = v;
            if (any_to) *cluster.map_shared_rank(abort_any, r) = 1;
          }
        }
      }
    }
    if (cl > 1) cluster.sync(); else __syncthreads();

    if (MODE == LOAD_STAGED) {
      if (*abort_any) {
        // A copy never completed: record it, wait (bounded) for the copies this
        // CTA still has in flight, and leave.  Every CTA of the cluster sees the
        // flag after the same barrier, so all of them leave together.
        if (tid == 0) {
          if (atomicCAS(p.status, 0, DEV_TIMEOUT) == 0) {
            *reinterpret_cast<volatile int64_t *>(p.status + 2) = row;
          }
          if (seg_len > 0) {
            for (int s = 0; s < stages; ++s) {
              const int64_t it2 = it + s;  // the ring's outstanding iterations
              const int64_t r2 = cluster_id + it2 * nclusters;
              if (r2 >= p.rows) break;
              mbar_wait_bounded(smem_addr(&bars[it2 % stages]),
                                static_cast<uint32_t>((it2 / stages) & 1));
            }
          }
        }
        if (cl > 1) cluster.sync(); else __syncthreads();
        return;
      }
      // every thread has read this stage: refill it with the row `stages` ahead
      if (tid == 0 && seg_len > 0) {
        const int64_t nrow = row + static_cast<int64_t>(stages) * nclusters;
        if (nrow < p.rows) issue(nrow, stage);
      }
    }

    double ss_row = 0.0;
    for (int i = lane; i < nslots; i += 32) ss_row = __dadd_rn(ss_row, ss_slots[i]);
    ss_row = warp_sum_d(ss_row);
    // Rms(x) = sqrt(ss/n + eps), fp64 as in the definition
    const double rms64 = __dsqrt_rn(
        __dadd_rn(__ddiv_rn(ss_row, static_cast<double>(n)), static_cast<double>(p.eps)));
    const float rinv32 = __frcp_rn(__double2float_rn(rms64));  // within 1 ulp of 1/Rms
    const float2 rinv2 = make_float2(rinv32, rinv32);

    // ---- pass 2: row max of |input_k|: binary32 scan, fp64 for the candidates
    double cand[NOUT];
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float m32 = 0.f;
#pragma unroll
      for (int k = 0; k < UPT; ++k)
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
          m32 = fmaxf(m32, fmaxf(fabsf(in.x), fabsf(in.y)));
        }
      // every element within the binary32 error bound of the thread's maximum is a
      // candidate for the true maximum; those are re-evaluated in fp64
      const float thr = m32 - 12.f * kUnit * (m32 + maxB[o]);
      double c64 = 0.0;
#pragma unroll
      for (int k = 0; k < UPT; ++k)
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
          if (fabsf(in.x) >= thr && m32 > 0.f)
            c64 = fmax(c64, fabs(input64(o, col(k, i, 0), xf[k][i].x, rms64)));
          if (fabsf(in.y) >= thr && m32 > 0.f)
            c64 = fmax(c64, fabs(input64(o, col(k, i, 1), xf[k][i].y, rms64)));
        }
      cand[o] = c64;
    }

    // ---- exchange 2: row max of |input_k| (fp64)
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      const double v = warp_max_d(cand[o]);
      if (lane == 0) {
        if (cl == 1) {
          max_slots[o * nslots + warp] = v;
        } else {
          for (int r = 0; r < cl; ++r)
            cluster.map_shared_rank(max_slots, r)[o * nslots + rank * nwarps + warp] = v;
        }
      }
    }
    if (cl > 1) cluster.sync(); else __syncthreads();

    // scale_k = fp32(row_max / Q); r = 1/scale (binary32); a zero scale gives zero
    // codes; a scale whose reciprocal is not a normal binary32 number sends every
    // code of the row through the fp64 path.
    float sc[NOUT], r32[NOUT], lim[NOUT];
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      double m = 0.0;
      for (int i = lane; i < nslots; i += 32) m = fmax(m, max_slots[o * nslots + i]);
      m = warp_max_d(m);
      sc[o] = __double2float_rn(__ddiv_rn(m, static_cast<double>(QI)));
      const bool tiny = sc[o] != 0.f && sc[o] < 1.1754943508222875e-38f;
      r32[o] = (sc[o] == 0.f || tiny) ? 0.f : __frcp_rn(sc[o]);
      // |t - t_exact| <= 10u (|t| + |B| r) (see the file header); 12u for margin,
      // plus the binary32 rounding of the scale itself
      const float tau = 12.f * kUnit * (QF + maxB[o] * r32[o]) + 2.f * kUnit * QF;
      lim[o] = tiny ? -1.f : 0.5f - tau;
      if (tid == 0 && rank == 0) p.scale[o][row] = sc[o];
    }

    // ---- pass 3: quantize (round half to even via the 1.5*2^23 trick) and store
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      const float2 r2 = make_float2(r32[o], r32[o]);
      uint8_t *y = p.y[o];
#pragma unroll
      for (int k = 0; k < UPT; ++k) {
        const int u = seg_begin + tid + k * static_cast<int>(blockDim.x);
        if (u >= seg_end) continue;
        uint32_t bits[2 * W];  // low bits: the code (two's complement)
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), G[o][k][i], B[o][k][i]);
          const float2 t = __fmul2_rn(in, r2);
          const float2 m = __fadd2_rn(t, make_float2(kMagic, kMagic));
          const float2 rr = __fadd2_rn(m, make_float2(-kMagic, -kMagic));  // RNE(t), exact
          const float2 d = __ffma2_rn(rr, make_float2(-1.f, -1.f), t);     // t - RNE(t), exact
          bits[2 * i] = __float_as_uint(m.x);
          bits[2 * i + 1] = __float_as_uint(m.y);
          const bool nx = fabsf(d.x) > lim[o];
          const bool ny = fabsf(d.y) > lim[o];
          if (nx || ny) {  // near a half-way point: decide in fp64
            const int h0 = nx ? 0 : 1, h1 = ny ? 1 : 0;
            for (int h = h0; h <= h1; ++h) {
              const float xv = h ? xf[k][i].y : xf[k][i].x;
              const double v = input64(o, col(k, i, h), xv, rms64);
              int q = 0;
              if (sc[o] != 0.f) {
                q = __double2int_rn(__ddiv_rn(v, static_cast<double>(sc[o])));
                q = min(max(q, -QI), QI);
              }
              bits[2 * i + h] = kMagicBits + static_cast<uint32_t>(q);
            }
          }
        }
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
      }
    }
  }
  // no CTA leaves while a peer may still touch its shared memory
  if (cl > 1) cluster.sync();
}

}  // namespace arnq
