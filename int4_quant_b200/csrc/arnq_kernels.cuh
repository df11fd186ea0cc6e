// arnq_kernels.cuh -- sm_100a kernels for the fused residual add + RMSNorm +
// per-row symmetric dynamic quantization operator (CANN page
// "aclnnAddRmsNormDynamicQuantV2", section "Formula"; the no-add form is the
// page "aclnnRmsNormDynamicQuant").
//
// One kernel template, three ways of bringing a row on chip:
//   LOAD_VEC     16-byte vector loads straight into registers (8 elements a unit)
//   LOAD_SCALAR  2-byte loads of element pairs, for misaligned tensors or n % 8 != 0
//   LOAD_STAGED  the CTA's slice of upcoming rows is copied into shared memory by
//                one thread with cp.async.bulk (1-D bulk copies, mbarrier
//                completion); a ring of `stages` rows keeps HBM reads in flight
//                while the threads work on the current row.
// A row is split over a thread-block cluster of `cl` CTAs when it is long or
// when there are too few rows to fill the SMs; partial sums and maxima are then
// exchanged through distributed shared memory.  Persistent grid: cluster c
// handles rows c, c + nclusters, ...
//
// Per row the work is: x = RNE16(fp32(x1) + fp32(x2)) -> xOut; ss = sum x^2
// (fp32, fixed tree); rinv = 1/sqrt(ss/n + eps); input_k = (x*rinv*gamma +
// beta) * smooth_k (fp32); amax_k = max |input_k|; scale_k = amax_k / Q;
// code = clamp(rint(input_k * (1/scale_k)), -Q, Q).  Two reductions, two
// barriers per row.  Nothing here is a contraction: no tensor cores.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace arnq {
namespace cg = cooperative_groups;

enum : int {
  F_X2 = 1,     // x2 given: x = x1 + x2 (else x = x1, the no-add operator)
  F_BETA = 2,
  F_S1 = 4,
  F_S2 = 8,
  F_OUT1 = 16,  // y1/scale1 selected
  F_OUT2 = 32,  // y2/scale2 selected
  F_XOUT = 64   // xOut written
};
enum : int { LOAD_VEC = 0, LOAD_SCALAR = 1, LOAD_STAGED = 2 };

// status codes the kernels record in the workspace status block
enum : int { DEV_TIMEOUT = 11 };

// A bounded wait gives up after this long (nanoseconds of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

struct KParams {
  const uint16_t *x1, *x2, *gamma, *beta, *s1, *s2;
  uint8_t *y1, *y2;
  float *scale1, *scale2;
  uint16_t *x_out;
  int32_t *status;      // workspace status block (staged kernel only; else unused)
  int64_t rows;
  int32_t n;            // row length in elements
  int32_t units;        // units per row: ceil(n / U)
  int32_t seg_units;    // units per CTA of a cluster
  int32_t flags;
  int32_t stages;       // staged kernel: ring depth
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
  static __device__ __forceinline__ uint16_t one(float v) {
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
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
  static __device__ __forceinline__ uint16_t one(float v) {
    __half h = __float2half_rn(v);
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ float2 warp_max2(float2 v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.x = fmaxf(v.x, __shfl_xor_sync(0xFFFFFFFFu, v.x, o));
    v.y = fmaxf(v.y, __shfl_xor_sync(0xFFFFFFFFu, v.y, o));
  }
  return v;
}

// ---------------------------------------------------------------- row kernel

// Threads per CTA the register budget allows: a thread keeps its UPT units of
// x (fp32) and of every parameter vector (packed 16-bit) across rows, so 8
// elements a thread fit in 64 registers (1024 threads) and 16 in 128 (512).
template <int MODE, int UPT>
struct MaxThreads {
  static constexpr int value = (UPT * (MODE == LOAD_SCALAR ? 2 : 8) <= 8) ? 1024 : 512;
};

template <class T, bool INT4, int MODE, int UPT>
__global__ void __launch_bounds__(MaxThreads<MODE, UPT>::value) rows_kernel(const KParams p) {
  using C = Cvt<T>;
  constexpr int U = (MODE == LOAD_SCALAR) ? 2 : 8;  // elements per unit
  constexpr int W = U / 2;                          // 32-bit words (element pairs) per unit
  constexpr float Q = INT4 ? 7.0f : 127.0f;
  constexpr int QI = INT4 ? 7 : 127;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int cl = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cluster_id = blockIdx.x / cl;
  const int64_t nclusters = gridDim.x / cl;
  const int flags = p.flags;
  const bool has_x2 = flags & F_X2;
  const int n = p.n;

  // ---- shared memory: [ss slots][amax slots][abort flag][mbarriers][stage ring]
  extern __shared__ __align__(128) unsigned char smem[];
  float *ss_slots = reinterpret_cast<float *>(smem);                 // cl * nwarps
  float2 *amax_slots = reinterpret_cast<float2 *>(smem + 16 * 32 * 4); // cl * nwarps
  int *abort_any = reinterpret_cast<int *>(smem + 16 * 32 * 4 + 16 * 32 * 8);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 16 * 32 * 12 + 128);
  unsigned char *ring = smem + 16 * 32 * 12 + 128 + 8 * 16;  // 16 mbarriers max; 128-aligned

  const int seg_begin = rank * p.seg_units;
  const int seg_end = min(seg_begin + p.seg_units, p.units);
  const int seg_len = max(seg_end - seg_begin, 0);
  const uint32_t seg_bytes = static_cast<uint32_t>(seg_len) * 16u;  // staged: bytes per input

  // ---- parameters for this thread's units, kept in registers for every row
  uint32_t gw[UPT][W], bw[UPT][W], s1w[UPT][W], s2w[UPT][W];
#pragma unroll
  for (int k = 0; k < UPT; ++k) {
    const int u = seg_begin + tid + k * blockDim.x;
    const bool ok = u < seg_end;
#pragma unroll
    for (int i = 0; i < W; ++i) gw[k][i] = bw[k][i] = s1w[k][i] = s2w[k][i] = 0u;
    if (!ok) continue;
    if (MODE != LOAD_SCALAR) {
      const uint4 g = ld_param16(p.gamma + static_cast<int64_t>(u) * 8);
      gw[k][0] = g.x; gw[k][1] = g.y; gw[k][2] = g.z; gw[k][3] = g.w;
      if (flags & F_BETA) {
        const uint4 b = ld_param16(p.beta + static_cast<int64_t>(u) * 8);
        bw[k][0] = b.x; bw[k][1] = b.y; bw[k][2] = b.z; bw[k][3] = b.w;
      }
      if (flags & F_S1) {
        const uint4 s = ld_param16(p.s1 + static_cast<int64_t>(u) * 8);
        s1w[k][0] = s.x; s1w[k][1] = s.y; s1w[k][2] = s.z; s1w[k][3] = s.w;
      }
      if (flags & F_S2) {
        const uint4 s = ld_param16(p.s2 + static_cast<int64_t>(u) * 8);
        s2w[k][0] = s.x; s2w[k][1] = s.y; s2w[k][2] = s.z; s2w[k][3] = s.w;
      }
    } else {
      const int j = 2 * u;
      const bool two = j + 1 < n;
      auto pair = [&](const uint16_t *a) -> uint32_t {
        uint32_t lo = __ldg(a + j);
        uint32_t hi = two ? __ldg(a + j + 1) : 0u;
        return lo | (hi << 16);
      };
      gw[k][0] = pair(p.gamma);
      if (flags & F_BETA) bw[k][0] = pair(p.beta);
      if (flags & F_S1) s1w[k][0] = pair(p.s1);
      if (flags & F_S2) s2w[k][0] = pair(p.s2);
    }
  }

  // ---- staged ring set-up
  uint64_t policy = 0;
  const int stages = (MODE == LOAD_STAGED) ? p.stages : 1;
  const uint32_t stage_stride = has_x2 ? 2u * seg_bytes : seg_bytes;
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
    if (has_x2) bulk_g2s(dst + seg_bytes, p.x2 + off, seg_bytes, bar, policy);
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

    // ---- pass 1: x = RNE16(x1 + x2) (or x1), xOut, sum of squares
    float xf[UPT][U];
    float2 ssv = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
      const int u = seg_begin + tid + k * blockDim.x;
      const bool ok = u < seg_end;
      uint32_t a[W], b[W];
#pragma unroll
      for (int i = 0; i < W; ++i) a[i] = b[i] = 0u;
      if (ok) {
        if (MODE == LOAD_VEC) {
          const int64_t off = row * n + static_cast<int64_t>(u) * 8;
          const uint4 va = ld_stream16(p.x1 + off);
          a[0] = va.x; a[1] = va.y; a[2] = va.z; a[3] = va.w;
          if (has_x2) {
            const uint4 vb = ld_stream16(p.x2 + off);
            b[0] = vb.x; b[1] = vb.y; b[2] = vb.z; b[3] = vb.w;
          }
        } else if (MODE == LOAD_STAGED) {
          const unsigned char *st = ring + static_cast<size_t>(stage) * stage_stride;
          const uint4 va = *reinterpret_cast<const uint4 *>(st + (u - seg_begin) * 16);
          a[0] = va.x; a[1] = va.y; a[2] = va.z; a[3] = va.w;
          if (has_x2) {
            const uint4 vb =
                *reinterpret_cast<const uint4 *>(st + seg_bytes + (u - seg_begin) * 16);
            b[0] = vb.x; b[1] = vb.y; b[2] = vb.z; b[3] = vb.w;
          }
        } else {
          const int64_t j = row * n + 2 * static_cast<int64_t>(u);
          const bool two = 2 * u + 1 < n;
          a[0] = static_cast<uint32_t>(__ldcs(p.x1 + j)) |
                 (two ? static_cast<uint32_t>(__ldcs(p.x1 + j + 1)) << 16 : 0u);
          if (has_x2)
            b[0] = static_cast<uint32_t>(__ldcs(p.x2 + j)) |
                   (two ? static_cast<uint32_t>(__ldcs(p.x2 + j + 1)) << 16 : 0u);
        }
      }
      uint32_t xo[W];
#pragma unroll
      for (int i = 0; i < W; ++i) {
        float2 xv;
        if (has_x2) {
          const float2 s = __fadd2_rn(C::f2(a[i]), C::f2(b[i]));  // binary32 add
          xo[i] = C::pack(s.x, s.y);                              // RNE to 16 bits
          xv = C::f2(xo[i]);                                      // x as normalised
        } else {
          xo[i] = a[i];
          xv = C::f2(a[i]);
        }
        xf[k][2 * i] = xv.x;
        xf[k][2 * i + 1] = xv.y;
        ssv = __ffma2_rn(xv, xv, ssv);
      }
      if (ok && (flags & F_XOUT)) {
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
      const float v = warp_sum(ssv.x + ssv.y);
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

    float ss;
    {
      float acc = 0.f;
      const int total = cl * nwarps;
      for (int i = lane; i < total; i += 32) acc += ss_slots[i];
      ss = warp_sum(acc);
    }
    // Rms(x) = sqrt(ss/n + eps); everything per row is IEEE-rounded binary32
    const float rinv = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(ss, static_cast<float>(n)),
                                                      p.eps)));
    const float2 rinv2 = make_float2(rinv, rinv);

    // ---- pass 2: input_k = (x*rinv*gamma + beta) * smooth_k; row max of |input_k|
    auto inputs = [&](int k, int i, float2 &in1, float2 &in2) {
      const float2 xv = make_float2(xf[k][2 * i], xf[k][2 * i + 1]);
      const float2 a = __fmul2_rn(xv, rinv2);
      float2 y;
      if (flags & F_BETA) y = __ffma2_rn(a, C::f2(gw[k][i]), C::f2(bw[k][i]));
      else y = __fmul2_rn(a, C::f2(gw[k][i]));
      in1 = (flags & F_S1) ? __fmul2_rn(y, C::f2(s1w[k][i])) : y;
      in2 = (flags & F_S2) ? __fmul2_rn(y, C::f2(s2w[k][i])) : y;
    };
    float2 amax = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        float2 in1, in2;
        inputs(k, i, in1, in2);
        amax.x = fmaxf(amax.x, fmaxf(fabsf(in1.x), fabsf(in1.y)));
        amax.y = fmaxf(amax.y, fmaxf(fabsf(in2.x), fabsf(in2.y)));
      }
    }

    // ---- exchange 2: row max of |input1| and |input2|
    {
      const float2 v = warp_max2(amax);
      if (lane == 0) {
        if (cl == 1) {
          amax_slots[warp] = v;
        } else {
          for (int r = 0; r < cl; ++r) cluster.map_shared_rank(amax_slots, r)[rank * nwarps + warp] = v;
        }
      }
    }
    if (cl > 1) cluster.sync(); else __syncthreads();
    {
      float2 acc = make_float2(0.f, 0.f);
      const int total = cl * nwarps;
      for (int i = lane; i < total; i += 32) {
        const float2 v = amax_slots[i];
        acc.x = fmaxf(acc.x, v.x);
        acc.y = fmaxf(acc.y, v.y);
      }
      amax = warp_max2(acc);
    }

    // scale_k = row_max / Q (binary32); codes use the reciprocal of that stored
    // scale.  A zero scale (all-zero row) gives all-zero codes; a scale too small
    // for its reciprocal to be finite divides element by element instead.
    const float sc1 = __fdiv_rn(amax.x, Q);
    const float sc2 = __fdiv_rn(amax.y, Q);
    const bool div1 = sc1 != 0.f && sc1 < 1.17549435e-38f;
    const bool div2 = sc2 != 0.f && sc2 < 1.17549435e-38f;
    const float r1 = (sc1 == 0.f) ? 0.f : __frcp_rn(sc1);
    const float r2 = (sc2 == 0.f) ? 0.f : __frcp_rn(sc2);
    if (tid == 0 && rank == 0) {
      if (flags & F_OUT1) p.scale1[row] = sc1;
      if (flags & F_OUT2) p.scale2[row] = sc2;
    }

    // ---- pass 3: quantize and store
    auto qcode = [&](float v, float r, float sc, bool dv) -> int {
      const float t = dv ? __fdiv_rn(v, sc) : __fmul_rn(v, r);
      const int q = __float2int_rn(t);  // round half to even
      return min(max(q, -QI), QI);
    };
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
      const int u = seg_begin + tid + k * blockDim.x;
      if (u >= seg_end) continue;
      uint32_t c1[W], c2[W];  // codes, packed per element pair (INT8: 2 bytes; INT4: 1 byte)
#pragma unroll
      for (int i = 0; i < W; ++i) {
        float2 in1, in2;
        inputs(k, i, in1, in2);
        const int a1 = qcode(in1.x, r1, sc1, div1), b1 = qcode(in1.y, r1, sc1, div1);
        const int a2 = qcode(in2.x, r2, sc2, div2), b2 = qcode(in2.y, r2, sc2, div2);
        if (INT4) {
          c1[i] = (static_cast<uint32_t>(a1) & 0xFu) | ((static_cast<uint32_t>(b1) & 0xFu) << 4);
          c2[i] = (static_cast<uint32_t>(a2) & 0xFu) | ((static_cast<uint32_t>(b2) & 0xFu) << 4);
        } else {
          c1[i] = (static_cast<uint32_t>(a1) & 0xFFu) | ((static_cast<uint32_t>(b1) & 0xFFu) << 8);
          c2[i] = (static_cast<uint32_t>(a2) & 0xFFu) | ((static_cast<uint32_t>(b2) & 0xFFu) << 8);
        }
      }
      auto store = [&](uint8_t *y, const uint32_t *c) {
        if (MODE != LOAD_SCALAR) {
          if (INT4) {  // 8 codes -> 4 bytes
            const uint32_t w = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
            __stcs(reinterpret_cast<unsigned int *>(y + row * (n / 2) + static_cast<int64_t>(u) * 4), w);
          } else {     // 8 codes -> 8 bytes
            const uint2 w = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
            __stcs(reinterpret_cast<uint2 *>(y + row * n + static_cast<int64_t>(u) * 8), w);
          }
        } else {
          if (INT4) {
            y[row * (n / 2) + u] = static_cast<uint8_t>(c[0]);
          } else {
            const int64_t j = row * n + 2 * static_cast<int64_t>(u);
            y[j] = static_cast<uint8_t>(c[0] & 0xFFu);
            if (2 * u + 1 < n) y[j + 1] = static_cast<uint8_t>(c[0] >> 8);
          }
        }
      };
      if (flags & F_OUT1) store(p.y1, c1);
      if (flags & F_OUT2) store(p.y2, c2);
    }
  }
  // no CTA leaves while a peer may still touch its shared memory
  if (cl > 1) cluster.sync();
}

}  // namespace arnq
