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
// A CTA is split into row groups that each work on their own rows and meet
// only at their own named barrier; the folded parameters live once per CTA in
// shared memory, so a thread's registers hold just its elements of x.
//
// Arithmetic.  The bulk of the work is binary32, two lanes at a time with the
// sm_100 packed instructions (add/mul/fma.rn.f32x2):
//   x = RNE16(x1 + x2)                    -> xOut, kept as fp32 in registers
//   ss = sum x^2                          fp64 (x^2 is exact; the sum agrees with
//                                         an fp64 evaluation of the definition)
//   rinv = 1/sqrt(ss/n + eps)             binary32, within 3 ulp
//   input_k = x*rinv*G_k + B_k            G_k = gamma*smooth_k, B_k = beta*smooth_k,
//                                         exact products of two 16-bit values
//   amax_k = max |input_k|                binary32 scan; the elements within the
//                                         error bound of the row maximum are
//                                         re-evaluated in fp64, so
//   scale_k = fp32(amax_k / Q)            equals the fp64 evaluation's scale
//   t = input_k * (1/scale_k)             rounded half-to-even by adding 1.5*2^23
// |t - t_exact| <= 7u|t| + 4u|B_k|/scale_k (u = 2^-24).  A code whose binary32
// quotient lies within that bound of a half-way point is recomputed in fp64 in
// the definition's order, (x / Rms * gamma + beta) * smooth / scale, so every
// rounding decision is the one an fp64 evaluation of the definition makes.
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
enum : int { DEV_TIMEOUT = 11 };

// A bounded wait gives up after this long (nanoseconds of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Shared-memory layout, sized by the launch (the host computes the same):
//   params   [NOUT][UPT][W][TG] float4 {G.x, G.y, B.x, B.y}: the folded
//            parameters of the CTA's columns, one copy shared by all groups
//   maxb     [NOUT][cl * warps per CTA] floats: set-up reduction of |B|
//   per row group g (stride `group`):
//     ss     [cl * warps per group] doubles: partial sums of squares
//     mx     [NOUT][cl * warps per group] floats: partial binary32 maxima
//     sc     [2][NOUT] binary32 bit patterns: the scales of the last two rows
//     abort  int; bars [stages] mbarriers; ring [stages] rows of staged input
constexpr int kMaxStagesDev = 8;
struct Layout {
  int params, maxb, group0, group;       // offsets and the per-group stride
  int ss, mx, sc, abort, bars, ring;     // offsets within a group
};
__host__ __device__ inline Layout make_layout(int groups, int tg, int pairs_per_thread, int nout,
                                              int cl, int stages, int stage_bytes) {
  Layout L;
  const int nwarps_cta = groups * tg / 32;
  const int nslots = cl * (tg / 32);
  int off = 0;
  L.params = off; off += nout * pairs_per_thread * tg * 16;
  L.maxb = off;   off += nout * cl * nwarps_cta * 4;
  L.group0 = (off + 127) & ~127;
  int g = 0;
  L.ss = g;    g += nslots * 8;
  L.mx = g;    g += nout * nslots * 4;
  L.sc = g;    g += 2 * nout * 4;
  g = (g + 7) & ~7;
  L.abort = g; g += 8;
  L.bars = g;  g += stages * 8;
  L.ring = (g + 127) & ~127;
  g = L.ring + stages * stage_bytes;
  L.group = (g + 127) & ~127;
  return L;
}
__host__ __device__ inline int layout_bytes(const Layout &L, int groups) {
  return L.group0 + groups * L.group;
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
  int32_t stages;             // staged kernel: ring depth per row group
  int32_t groups;             // row groups per CTA (1 when cl > 1)
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
// Threads per CTA: 512, so a thread may use 128 registers -- x for up to 32
// elements plus the fp64 paths, without spilling.
template <int MODE, int UPT>
struct MaxThreads {
  static constexpr int value = 512;
};

constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: v + kMagic = RNE(v) + kMagic
constexpr uint32_t kMagicBits = 0x4B400000u;  // its bit pattern; low bits then hold RNE(v)
constexpr float kUnit = 5.9604644775390625e-08f;  // 2^-24, binary32 unit roundoff

// Rms(x) = sqrt(ss/n + eps) in fp64, IEEE-rounded operations in the
// definition's order.
static __device__ __forceinline__ double rms_exact(double ss, int n, float eps) {
  return __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(n)), static_cast<double>(eps)));
}

// |input| of one element in fp64 from the folded parameters, which are exact
// products (G = gamma*smooth, B = beta*smooth fit in binary32): |x/Rms*G + B|.
static __device__ __forceinline__ double input_abs_folded(float x, float g, float b, double rms) {
  return fabs(__fma_rn(__ddiv_rn(static_cast<double>(x), rms), static_cast<double>(g),
                       static_cast<double>(b)));
}

// The code of one element decided in fp64 exactly as the definition orders it:
// round_half_even((x / Rms * gamma + beta) * smooth / scale), clamped to
// [-Q, Q]; returned as kMagicBits + code so its low bits pack like the fast path.
template <class T>
__device__ __forceinline__ uint32_t code_exact(const uint16_t *gamma, const uint16_t *beta,
                                            const uint16_t *smooth, int c, float x, double rms,
                                            float scale, int qmax) {
  int q = 0;
  if (scale != 0.f) {
    double y = __dmul_rn(__ddiv_rn(static_cast<double>(x), rms),
                         static_cast<double>(Cvt<T>::f1(gamma[c])));
    if (beta) y = __dadd_rn(y, static_cast<double>(Cvt<T>::f1(beta[c])));
    if (smooth) y = __dmul_rn(y, static_cast<double>(Cvt<T>::f1(smooth[c])));
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

// ---------------------------------------------------------------- row kernel

// A CTA holds `groups` row groups of TG = blockDim / groups threads.  Each group
// works on its own rows (group id g of cluster c takes rows c*groups + g,
// + nclusters*groups, ...) and synchronizes only its own threads, with the
// named barrier 1 + g; a cluster (cl > 1) has one group per CTA and uses the
// cluster barrier.
template <class T, bool INT4, int MODE, int UPT, int NOUT, bool ADD>
__global__ void __launch_bounds__(MaxThreads<MODE, UPT>::value) rows_kernel(const KParams p) {
  using C = Cvt<T>;
  constexpr int U = (MODE == LOAD_SCALAR) ? 2 : 8;  // elements per unit
  constexpr int W = U / 2;                          // element pairs per unit
  constexpr int QI = INT4 ? 7 : 127;
  constexpr float QF = static_cast<float>(QI);
  constexpr int NIN = ADD ? 2 : 1;                  // staged inputs per row

  cg::cluster_group cluster = cg::this_cluster();
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cluster_id = blockIdx.x / cl;
  const int64_t nclusters = gridDim.x / cl;
  const int groups = p.groups;
  const int TG = static_cast<int>(blockDim.x) / groups;
  const int tid = threadIdx.x;
  const int gid = tid / TG;           // row group
  const int gt = tid - gid * TG;      // thread within the group
  const int lane = tid & 31;
  const int gwarp = gt >> 5;
  const int nwg = TG >> 5;            // warps per group
  const int nslots = cl * nwg;
  const int my_slot = rank * nwg + gwarp;
  const int64_t group_id = cluster_id * groups + gid;
  const int64_t ngroups = nclusters * groups;
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
  const Layout lay = make_layout(groups, TG, UPT * W, NOUT, cl, ring_depth, stage_bytes);
  float4 *params = reinterpret_cast<float4 *>(smem + lay.params);
  float *maxb_slots = reinterpret_cast<float *>(smem + lay.maxb);
  unsigned char *gb = smem + lay.group0 + gid * lay.group;
  double *ss_slots = reinterpret_cast<double *>(gb + lay.ss);   // [nslots]
  float *mx_slots = reinterpret_cast<float *>(gb + lay.mx);     // [NOUT][nslots]
  unsigned *sc_slot = reinterpret_cast<unsigned *>(gb + lay.sc);  // [2][NOUT]
  int *abort_flag = reinterpret_cast<int *>(gb + lay.abort);
  uint64_t *bars = reinterpret_cast<uint64_t *>(gb + lay.bars);
  unsigned char *ring = gb + lay.ring;

  auto group_sync = [&]() {
    if (cl > 1) {
      cluster.sync();
    } else {
      asm volatile("bar.sync %0, %1;" ::"r"(1 + gid), "r"(TG) : "memory");
    }
  };
  // the folded parameters of pair i of this thread's k-th unit, output o
  auto par = [&](int o, int k, int i) -> float4 {
    return params[((o * UPT + k) * W + i) * TG + gt];
  };

  // ---- set-up: fold gamma, beta, smooth into G, B (group 0 writes the shared
  // copy); every thread keeps the bound on |B| over its own elements
  float maxB[NOUT];
#pragma unroll
  for (int o = 0; o < NOUT; ++o) maxB[o] = 0.f;
#pragma unroll
  for (int k = 0; k < UPT; ++k) {
    const int u = seg_begin + gt + k * TG;
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
        const float2 G = __fmul2_rn(g2, s2);  // exact: two 8- (or 11-) bit significands
        const float2 B = __fmul2_rn(b2, s2);
        maxB[o] = fmaxf(maxB[o], fmaxf(fabsf(B.x), fabsf(B.y)));
        if (gid == 0) params[((o * UPT + k) * W + i) * TG + gt] = make_float4(G.x, G.y, B.x, B.y);
      }
    }
  }
  const int nwarps_cta = static_cast<int>(blockDim.x) >> 5;
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    const float v = warp_max_nonneg(maxB[o]);
    if (lane == 0) {
      const int slot = o * cl * nwarps_cta + rank * nwarps_cta + (tid >> 5);
      if (cl == 1) {
        maxb_slots[slot] = v;
      } else {
        for (int r = 0; r < cl; ++r) cluster.map_shared_rank(maxb_slots, r)[slot] = v;
      }
    }
  }
  if (gt == 0) {
    *abort_flag = 0;
    for (int q = 0; q < 2 * NOUT; ++q) sc_slot[q] = 0u;
    if (MODE == LOAD_STAGED) {
      for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  if (cl > 1) cluster.sync(); else __syncthreads();
  float maxBg[NOUT];  // bound on |B| over the whole row
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    float m = 0.f;
    for (int i = lane; i < cl * nwarps_cta; i += 32) m = fmaxf(m, maxb_slots[o * cl * nwarps_cta + i]);
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
  if (MODE == LOAD_STAGED && gt == 0 && seg_len > 0) {
    policy = policy_evict_first();
    for (int s = 0; s < stages; ++s) {
      const int64_t row = group_id + s * ngroups;
      if (row < p.rows) issue(row, s);
    }
  }

  int64_t it = 0;
  for (int64_t row = group_id; row < p.rows; row += ngroups, ++it) {
    const int stage = (MODE == LOAD_STAGED) ? static_cast<int>(it % stages) : 0;
    const int par2 = static_cast<int>(it & 1);
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
      const int u = seg_begin + gt + k * TG;
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
        if (cl == 1) {
          ss_slots[gwarp] = v;
          if (any_to) *abort_flag = 1;
        } else {
          for (int r = 0; r < cl; ++r) {
            cluster.map_shared_rank(ss_slots, r)[my_slot] = v;
            if (any_to) *cluster.map_shared_rank(abort_flag, r) = 1;
          }
        }
      }
    }
    group_sync();

    if (MODE == LOAD_STAGED) {
      if (*abort_flag) {
        // A copy never completed: record it, wait (bounded) for the copies this
        // group still has in flight, and stop.  Every thread of the group (and
        // of the cluster) sees the flag after the same barrier.
        if (gt == 0) {
          if (atomicCAS(p.status, 0, DEV_TIMEOUT) == 0) {
            *reinterpret_cast<volatile int64_t *>(p.status + 2) = row;
          }
          if (seg_len > 0) {
            for (int s = 0; s < stages; ++s) {
              const int64_t it2 = it + s;  // the ring's outstanding iterations
              if (group_id + it2 * ngroups >= p.rows) break;
              mbar_wait_bounded(smem_addr(&bars[it2 % stages]),
                                static_cast<uint32_t>((it2 / stages) & 1));
            }
          }
        }
        break;
      }
      // every thread of the group has read this stage: refill it
      if (gt == 0 && seg_len > 0) {
        const int64_t nrow = row + static_cast<int64_t>(stages) * ngroups;
        if (nrow < p.rows) issue(nrow, stage);
      }
    }
    // every thread read the previous row's scales before this barrier
    if (gt == 0) {
#pragma unroll
      for (int o = 0; o < NOUT; ++o) sc_slot[(par2 ^ 1) * NOUT + o] = 0u;
    }

    double ss_row = 0.0;
    for (int i = lane; i < nslots; i += 32) ss_row = __dadd_rn(ss_row, ss_slots[i]);
    ss_row = warp_sum_d(ss_row);
    float2 rinv2;
    {
      const float v = __double2float_rn(__fma_rn(ss_row, p.inv_n, static_cast<double>(p.eps)));
      const float r = rsqrt_refined(v);
      rinv2 = make_float2(r, r);
    }

    // ---- pass 2: binary32 row maxima of |input_k|
    float m32[NOUT];
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < UPT; ++k)
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float4 gbv = par(o, k, i);
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), make_float2(gbv.x, gbv.y),
                                       make_float2(gbv.z, gbv.w));
          m = fmaxf(m, fmaxf(fabsf(in.x), fabsf(in.y)));
        }
      m32[o] = m;
      const float v = warp_max_nonneg(m);
      if (lane == 0) {
        if (cl == 1) {
          mx_slots[o * nslots + gwarp] = v;
        } else {
          for (int r = 0; r < cl; ++r) cluster.map_shared_rank(mx_slots, r)[o * nslots + my_slot] = v;
        }
      }
    }
    // ---- exchange 2: binary32 row maxima
    group_sync();

    // Every element whose binary32 value is within the error bound of the row
    // maximum is a candidate for the true maximum (usually exactly one per row).
    // Candidates are evaluated in fp64 and each offers fp32(|input| / Q); as that
    // rounding is monotonic, the atomic maximum of the offers (binary32 bit
    // patterns of non-negative values order as integers) is fp32(amax / Q).
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      float g = 0.f;
      for (int i = lane; i < nslots; i += 32) g = fmaxf(g, mx_slots[o * nslots + i]);
      g = warp_max_nonneg(g);
      const float thr = g - 12.f * kUnit * (g + maxBg[o]);
      if (g > 0.f && m32[o] >= thr) {
        const double rms = rms_exact(ss_row, n, p.eps);
        double c64 = 0.0;
#pragma unroll
        for (int k = 0; k < UPT; ++k)
#pragma unroll
          for (int i = 0; i < W; ++i) {
            const float4 gbv = par(o, k, i);
            const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), make_float2(gbv.x, gbv.y),
                                         make_float2(gbv.z, gbv.w));
            if (fabsf(in.x) >= thr)
              c64 = fmax(c64, input_abs_folded(xf[k][i].x, gbv.x, gbv.z, rms));
            if (fabsf(in.y) >= thr)
              c64 = fmax(c64, input_abs_folded(xf[k][i].y, gbv.y, gbv.w, rms));
          }
        const unsigned offer =
            __float_as_uint(__double2float_rn(__ddiv_rn(c64, static_cast<double>(QI))));
        unsigned *slot = &sc_slot[par2 * NOUT + o];
        if (cl == 1) {
          atomicMax(slot, offer);
        } else {
          for (int r = 0; r < cl; ++r) atomicMax(cluster.map_shared_rank(slot, r), offer);
        }
      }
    }
    // ---- exchange 3: the scales
    group_sync();

    // ---- pass 3: quantize (round half to even via the 1.5*2^23 trick) and store.
    // A zero scale gives zero codes; a scale whose reciprocal is not a normal
    // binary32 number sends every code of the row through the fp64 path.
    double rms_cached = -1.0;
#pragma unroll
    for (int o = 0; o < NOUT; ++o) {
      const float sc = __uint_as_float(sc_slot[par2 * NOUT + o]);
      const bool tiny = sc != 0.f && sc < 1.1754943508222875e-38f;
      const float r32 = (sc == 0.f || tiny) ? 0.f : __frcp_rn(sc);
      const float tau = 12.f * kUnit * (QF + maxB[o] * r32) + 2.f * kUnit * QF;
      const float lim = tiny ? -1.f : 0.5f - tau;
      if (gt == 0 && rank == 0) p.scale[o][row] = sc;
      const float2 r2 = make_float2(r32, r32);
      uint8_t *y = p.y[o];
#pragma unroll
      for (int k = 0; k < UPT; ++k) {
        const int u = seg_begin + gt + k * TG;
        if (u >= seg_end) continue;
        uint32_t bits[2 * W];  // low bits: the code (two's complement)
        float dmax = 0.f;      // largest |t - RNE(t)| of the unit
#pragma unroll
        for (int i = 0; i < W; ++i) {
          const float4 gbv = par(o, k, i);
          const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), make_float2(gbv.x, gbv.y),
                                       make_float2(gbv.z, gbv.w));
          const float2 t = __fmul2_rn(in, r2);
          const float2 m = __fadd2_rn(t, make_float2(kMagic, kMagic));
          const float2 rr = __fadd2_rn(m, make_float2(-kMagic, -kMagic));  // RNE(t), exact
          const float2 d = __ffma2_rn(rr, make_float2(-1.f, -1.f), t);     // t - RNE(t), exact
          bits[2 * i] = __float_as_uint(m.x);
          bits[2 * i + 1] = __float_as_uint(m.y);
          dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        }
        if (dmax > lim) {  // some code is near a half-way point: decide those in fp64
          if (rms_cached < 0.0) rms_cached = rms_exact(ss_row, n, p.eps);
#pragma unroll
          for (int i = 0; i < W; ++i) {
            const float4 gbv = par(o, k, i);
            const float2 in = __ffma2_rn(__fmul2_rn(xf[k][i], rinv2), make_float2(gbv.x, gbv.y),
                                         make_float2(gbv.z, gbv.w));
            const float2 t = __fmul2_rn(in, r2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float th = h ? t.y : t.x;
              const float dv = fabsf(th - rintf(th));
              if (dv > lim)
                bits[2 * i + h] = code_exact<T>(p.gamma, has_beta ? p.beta : nullptr,
                                                p.smooth[o], u * U + 2 * i + h,
                                                h ? xf[k][i].y : xf[k][i].x, rms_cached, sc, QI);
            }
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
