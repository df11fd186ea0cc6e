// arnq_api.cu -- host side of the C ABI declared in include/arnq.h: argument
// validation (the "Constraints" section of the CANN page
// "aclnnAddRmsNormDynamicQuantV2" plus the library's own shape / alignment /
// workspace rules), launch-plan selection and the kernel launch.
//
// Every check runs before any CUDA call, so a rejected call touches no device.
// Nothing here allocates device memory or synchronizes.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "arnq.h"
#include "arnq_kernels.cuh"

namespace {

using arnq::KParams;
typedef void (*KernelFn)(KParams);

constexpr int kHeaderSmem = 16 * 32 * 12 + 128 + 8 * 16;  // slots, abort flag, mbarriers
constexpr size_t kWorkspaceBytes = 256;                     // status block, padded
constexpr int kMaxStages = 16;
constexpr int kMaxCluster = 16;

// ---------------------------------------------------------------- kernel table

constexpr int kUptSlots = 4;  // units per thread 1, 2, 4, 8
int upt_slot(int upt) { return upt == 1 ? 0 : upt == 2 ? 1 : upt == 4 ? 2 : upt == 8 ? 3 : -1; }

template <class T, bool I4, int M>
void fill_mode(KernelFn *t) {
  t[0] = arnq::rows_kernel<T, I4, M, 1>;
  t[1] = arnq::rows_kernel<T, I4, M, 2>;
  if (M == arnq::LOAD_SCALAR) {
    t[2] = arnq::rows_kernel<T, I4, arnq::LOAD_SCALAR, 4>;
    t[3] = arnq::rows_kernel<T, I4, arnq::LOAD_SCALAR, 8>;
  } else {
    t[2] = t[3] = nullptr;  // vector units: at most 2 per thread (register budget)
  }
}

template <class T, bool I4>
void fill_q(KernelFn *t) {
  fill_mode<T, I4, arnq::LOAD_VEC>(t + 0 * kUptSlots);
  fill_mode<T, I4, arnq::LOAD_SCALAR>(t + 1 * kUptSlots);
  fill_mode<T, I4, arnq::LOAD_STAGED>(t + 2 * kUptSlots);
}

struct KernelTable {
  KernelFn fn[2][2][3 * kUptSlots];
  KernelTable() {
    fill_q<arnq::Bf16, false>(fn[0][0]);
    fill_q<arnq::Bf16, true>(fn[0][1]);
    fill_q<arnq::Fp16, false>(fn[1][0]);
    fill_q<arnq::Fp16, true>(fn[1][1]);
  }
};

KernelFn lookup(int dt, int qdt, int mode, int upt) {
  static const KernelTable table;
  const int s = upt_slot(upt);
  if (s < 0) return nullptr;
  return table.fn[dt][qdt][mode * kUptSlots + s];
}

// ---------------------------------------------------------------- device info

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int smem_per_block_optin = 0;
  int smem_per_sm = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

struct AttrKey {
  KernelFn fn;
  int dev;
  int smem;
};
constexpr int kMaxAttrKeys = 512;
AttrKey g_attr[kMaxAttrKeys];
int g_nattr = 0;

arnq_status device_info(DeviceInfo *out, int *dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ARNQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ARNQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_per_block_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                               dev) != cudaSuccess)
      return ARNQ_ERR_CUDA;
    d.ready = true;
  }
  *out = d;
  *dev_out = dev;
  return ARNQ_OK;
}

// Raises the kernel's dynamic shared memory limit (and allows 16-CTA clusters)
// once per kernel, device and size.
arnq_status prepare_kernel(KernelFn fn, int dev, int smem) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_nattr; ++i)
    if (g_attr[i].fn == fn && g_attr[i].dev == dev && g_attr[i].smem >= smem) return ARNQ_OK;
  if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ARNQ_ERR_CUDA;
  if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn),
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return ARNQ_ERR_CUDA;
  for (int i = 0; i < g_nattr; ++i)
    if (g_attr[i].fn == fn && g_attr[i].dev == dev) {
      g_attr[i].smem = smem;
      return ARNQ_OK;
    }
  if (g_nattr < kMaxAttrKeys) g_attr[g_nattr++] = AttrKey{fn, dev, smem};
  return ARNQ_OK;
}

// ---------------------------------------------------------------- validation

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Problem {
  const void *x1, *x2, *gamma, *beta, *s1, *s2;
  void *y1, *y2, *x_out;
  float *scale1, *scale2;
  int64_t rows, n;
  int dt, qdt;
  float eps;
  int flags;
};

arnq_status selected(int out_mask, int has_s1, int has_s2, int *on1, int *on2) {
  if (out_mask != ARNQ_MASK_ABSENT && (out_mask < 0 || out_mask > 3)) return ARNQ_ERR_MASK;
  const bool present = out_mask != ARNQ_MASK_ABSENT;
  const bool m0 = present && (out_mask & ARNQ_MASK_Y1);
  const bool m1 = present && (out_mask & ARNQ_MASK_Y2);
  // Constraints: mask given with smoothScale1 -> mask[0]; with smoothScale2 -> mask[1];
  // mask entries not both false; no mask with smoothScale2 -> smoothScale1 given.
  if (present && has_s1 && !m0) return ARNQ_ERR_MASK;
  if (present && has_s2 && !m1) return ARNQ_ERR_MASK;
  if (present && !m0 && !m1) return ARNQ_ERR_MASK;
  if (!present && has_s2 && !has_s1) return ARNQ_ERR_MASK;
  // Formula: y1Out valid with mask[0] or no mask; y2Out valid with mask[1] or
  // (no mask and both smooth scales).
  if (on1) *on1 = (m0 || !present) ? 1 : 0;
  if (on2) *on2 = (m1 || (!present && has_s1 && has_s2)) ? 1 : 0;
  return ARNQ_OK;
}

arnq_status check_shape(int64_t rows, int64_t n, int dt, int qdt, float eps) {
  if (dt != ARNQ_BF16 && dt != ARNQ_FP16) return ARNQ_ERR_DTYPE;
  if (qdt != ARNQ_INT8 && qdt != ARNQ_INT4) return ARNQ_ERR_DTYPE;
  if (rows < 0 || n < 0) return ARNQ_ERR_SHAPE;
  if (rows == 0 || n == 0) return ARNQ_ERR_EMPTY;
  if (n > ARNQ_MAX_N) return ARNQ_ERR_SHAPE;
  if (qdt == ARNQ_INT4 && (n % 2) != 0) return ARNQ_ERR_SHAPE;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return ARNQ_ERR_EPS;
  return ARNQ_OK;
}

// Validates a problem; `has_add` false for the no-add operator (x2 unused).
arnq_status validate(const Problem &P, bool has_add, int out_mask, const void *workspace,
                     size_t workspace_bytes, int *flags_out) {
  arnq_status st = check_shape(P.rows, P.n, P.dt, P.qdt, P.eps);
  if (st != ARNQ_OK) return st;
  int on1 = 0, on2 = 0;
  st = selected(out_mask, P.s1 != nullptr, P.s2 != nullptr, &on1, &on2);
  if (st != ARNQ_OK) return st;
  if (!P.x1 || (has_add && !P.x2) || !P.gamma) return ARNQ_ERR_NULL_PTR;
  if (on1 && (!P.y1 || !P.scale1)) return ARNQ_ERR_NULL_PTR;
  if (on2 && (!P.y2 || !P.scale2)) return ARNQ_ERR_NULL_PTR;
  const void *h16[] = {P.x1, has_add ? P.x2 : nullptr, P.gamma, P.beta, P.s1, P.s2, P.x_out};
  for (const void *q : h16)
    if (q && !aligned(q, 2)) return ARNQ_ERR_ALIGN;
  if ((on1 && !aligned(P.scale1, 4)) || (on2 && !aligned(P.scale2, 4))) return ARNQ_ERR_ALIGN;
  if (!workspace || workspace_bytes < kWorkspaceBytes) return ARNQ_ERR_WORKSPACE;
  if (!aligned(workspace, 8)) return ARNQ_ERR_ALIGN;
  int f = 0;
  if (has_add) f |= arnq::F_X2;
  if (P.beta) f |= arnq::F_BETA;
  if (P.s1) f |= arnq::F_S1;
  if (P.s2) f |= arnq::F_S2;
  if (on1) f |= arnq::F_OUT1;
  if (on2) f |= arnq::F_OUT2;
  if (has_add && P.x_out) f |= arnq::F_XOUT;
  *flags_out = f;
  return ARNQ_OK;
}

// ---------------------------------------------------------------- planning

int round_up(int v, int m) { return (v + m - 1) / m * m; }
int max_threads(int mode, int upt) {
  return upt * (mode == arnq::LOAD_SCALAR ? 2 : 8) <= 8 ? 1024 : 512;
}
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool vector_ok(const Problem &P) {
  if (P.n % 8 != 0) return false;
  const bool x2 = (P.flags & arnq::F_X2) != 0;
  const void *v16[] = {P.x1, x2 ? P.x2 : nullptr, P.gamma, P.beta, P.s1, P.s2,
                       (P.flags & arnq::F_XOUT) ? P.x_out : nullptr};
  for (const void *q : v16)
    if (q && !aligned(q, 16)) return false;
  const uintptr_t ya = (P.qdt == ARNQ_INT8) ? 8 : 4;
  if ((P.flags & arnq::F_OUT1) && !aligned(P.y1, ya)) return false;
  if ((P.flags & arnq::F_OUT2) && !aligned(P.y2, ya)) return false;
  return true;
}

int stage_smem(const arnq_plan &pl, int seg_units, bool x2) {
  return kHeaderSmem + pl.stages * seg_units * 16 * (x2 ? 2 : 1);
}

arnq_status make_plan(const Problem &P, arnq_plan *pl, KernelFn *fn_out, int *smem_out,
                      int *seg_out, int *units_out) {
  DeviceInfo di;
  int dev = 0;
  arnq_status st = device_info(&di, &dev);
  if (st != ARNQ_OK) return st;
  const bool vec = vector_ok(P);
  const bool x2 = (P.flags & arnq::F_X2) != 0;
  if (pl->kernel == ARNQ_KERNEL_AUTO) pl->kernel = vec ? ARNQ_KERNEL_STAGED : ARNQ_KERNEL_DIRECT;
  if (pl->kernel == ARNQ_KERNEL_STAGED && !vec) return ARNQ_ERR_PLAN;
  if (pl->kernel != ARNQ_KERNEL_DIRECT && pl->kernel != ARNQ_KERNEL_STAGED) return ARNQ_ERR_PLAN;
  const int mode = pl->kernel == ARNQ_KERNEL_STAGED ? arnq::LOAD_STAGED
                   : vec                            ? arnq::LOAD_VEC
                                                    : arnq::LOAD_SCALAR;
  pl->vector = (mode != arnq::LOAD_SCALAR) ? 1 : 0;
  const int U = (mode == arnq::LOAD_SCALAR) ? 2 : 8;
  const int units = static_cast<int>(ceil_div(P.n, U));
  const int max_upt = (mode == arnq::LOAD_SCALAR) ? 8 : 2;

  // cluster: enough CTAs per row that one CTA's slice fits, then spread rows
  // that are too few to fill the SMs over more CTAs
  // a CTA holds at most 8192 elements of a row in registers (see MaxThreads)
  const int max_seg = 8192 / U;
  if (pl->cluster == 0) {
    int cl = 1;
    while (cl < kMaxCluster && ceil_div(units, cl) > max_seg) cl *= 2;
    while (cl < kMaxCluster && P.rows * cl < di.sms && ceil_div(units, 2 * cl) >= 64) cl *= 2;
    pl->cluster = cl;
  }
  const int cl = pl->cluster;
  if (cl != 1 && cl != 2 && cl != 4 && cl != 8 && cl != 16) return ARNQ_ERR_PLAN;
  const int seg = static_cast<int>(ceil_div(units, cl));

  if (seg > max_seg) return ARNQ_ERR_PLAN;
  if (pl->units == 0) {
    int upt = 1;
    while (upt < max_upt && ceil_div(seg, upt) > max_threads(mode, upt)) upt *= 2;
    while (upt < max_upt && ceil_div(seg, upt) > 512 && U * upt * 2 <= 8) upt *= 2;
    pl->units = upt;
  }
  if (pl->units > max_upt || upt_slot(pl->units) < 0) return ARNQ_ERR_PLAN;
  if (pl->threads == 0) {
    pl->threads = round_up(static_cast<int>(ceil_div(seg, pl->units)), 32);
    if (pl->threads < 32) pl->threads = 32;
  }
  if (pl->threads % 32 != 0 || pl->threads > max_threads(mode, pl->units) ||
      static_cast<int64_t>(pl->threads) * pl->units < seg)
    return ARNQ_ERR_PLAN;

  KernelFn fn = lookup(P.dt, P.qdt, mode, pl->units);
  if (!fn) return ARNQ_ERR_PLAN;

  int smem = kHeaderSmem;
  if (mode == arnq::LOAD_STAGED) {
    if (pl->ctas_per_sm == 0) pl->ctas_per_sm = 2;
    if (pl->stages == 0) {
      const int budget = di.smem_per_sm / pl->ctas_per_sm - 1024;  // 1 KB reserved per CTA
      const int cap = budget < di.smem_per_block_optin ? budget : di.smem_per_block_optin;
      const int per_stage = seg * 16 * (x2 ? 2 : 1);
      int s = (cap - kHeaderSmem) / per_stage;
      if (s > kMaxStages) s = kMaxStages;
      if (s < 1) s = 1;
      pl->stages = s;
    }
    if (pl->stages < 1 || pl->stages > kMaxStages) return ARNQ_ERR_PLAN;
    smem = stage_smem(*pl, seg, x2);
    if (smem > di.smem_per_block_optin) return ARNQ_ERR_PLAN;
  } else {
    pl->stages = 0;
  }
  st = prepare_kernel(fn, dev, smem);
  if (st != ARNQ_OK) return st;

  // grid: persistent, as many clusters as fit at once (or one per row)
  int64_t clusters_needed = P.rows;
  int64_t clusters_fit = 0;
  if (cl == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, pl->threads, smem) !=
        cudaSuccess)
      return ARNQ_ERR_CUDA;
    if (per_sm < 1) return ARNQ_ERR_PLAN;
    if (pl->ctas_per_sm != 0 && pl->ctas_per_sm < per_sm) per_sm = pl->ctas_per_sm;
    if (pl->ctas_per_sm == 0) pl->ctas_per_sm = per_sm;
    clusters_fit = static_cast<int64_t>(per_sm) * di.sms;
  } else {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(cl * 1024, 1, 1);
    cfg.blockDim = dim3(pl->threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, fn, &cfg) != cudaSuccess) return ARNQ_ERR_CUDA;
    if (nc < 1) return ARNQ_ERR_PLAN;
    int64_t want = pl->ctas_per_sm != 0 ? static_cast<int64_t>(pl->ctas_per_sm) * di.sms / cl : nc;
    if (want < 1) want = 1;
    clusters_fit = want < nc ? want : nc;
    if (pl->ctas_per_sm == 0) pl->ctas_per_sm = static_cast<int32_t>(ceil_div(nc * cl, di.sms));
  }
  const int64_t nclusters = clusters_needed < clusters_fit ? clusters_needed : clusters_fit;
  pl->grid = static_cast<int32_t>(nclusters * cl);
  *fn_out = fn;
  *smem_out = smem;
  *seg_out = seg;
  *units_out = units;
  return ARNQ_OK;
}

arnq_status launch(const Problem &P, arnq_plan plan, void *workspace, cudaStream_t stream) {
  KernelFn fn = nullptr;
  int smem = 0, seg = 0, units = 0;
  arnq_status st = make_plan(P, &plan, &fn, &smem, &seg, &units);
  if (st != ARNQ_OK) return st;
  KParams k;
  k.x1 = static_cast<const uint16_t *>(P.x1);
  k.x2 = static_cast<const uint16_t *>(P.x2);
  k.gamma = static_cast<const uint16_t *>(P.gamma);
  k.beta = static_cast<const uint16_t *>(P.beta);
  k.s1 = static_cast<const uint16_t *>(P.s1);
  k.s2 = static_cast<const uint16_t *>(P.s2);
  k.y1 = static_cast<uint8_t *>(P.y1);
  k.y2 = static_cast<uint8_t *>(P.y2);
  k.scale1 = P.scale1;
  k.scale2 = P.scale2;
  k.x_out = static_cast<uint16_t *>(P.x_out);
  k.status = static_cast<int32_t *>(workspace);
  k.rows = P.rows;
  k.n = static_cast<int32_t>(P.n);
  k.units = units;
  k.seg_units = seg;
  k.flags = P.flags;
  k.stages = plan.stages;
  k.eps = P.eps;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  if (plan.cluster > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  if (cudaLaunchKernelEx(&cfg, fn, k) != cudaSuccess) return ARNQ_ERR_CUDA;
  return ARNQ_OK;
}

Problem problem(const void *x1, const void *x2, const void *gamma, const void *beta,
                const void *s1, const void *s2, int64_t rows, int64_t n, arnq_dtype dt,
                float eps, arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                void *x_out) {
  Problem P;
  P.x1 = x1; P.x2 = x2; P.gamma = gamma; P.beta = beta; P.s1 = s1; P.s2 = s2;
  P.y1 = y1; P.y2 = y2; P.x_out = x_out; P.scale1 = scale1; P.scale2 = scale2;
  P.rows = rows; P.n = n; P.dt = static_cast<int>(dt); P.qdt = static_cast<int>(qdt);
  P.eps = eps; P.flags = 0;
  return P;
}

arnq_status run_common(Problem P, bool has_add, int out_mask, void *workspace,
                       size_t workspace_bytes, void *stream, const arnq_plan *plan) {
  int flags = 0;
  arnq_status st = validate(P, has_add, out_mask, workspace, workspace_bytes, &flags);
  if (st != ARNQ_OK) return st;
  P.flags = flags;
  if (!(flags & arnq::F_OUT1)) { P.y1 = nullptr; P.scale1 = nullptr; }
  if (!(flags & arnq::F_OUT2)) { P.y2 = nullptr; P.scale2 = nullptr; }
  if (!has_add) { P.x2 = nullptr; P.x_out = nullptr; }
  arnq_plan pl;
  std::memset(&pl, 0, sizeof pl);
  if (plan) pl = *plan;
  return launch(P, pl, workspace, static_cast<cudaStream_t>(stream));
}

}  // namespace

// ============================================================== C ABI

extern "C" {

const char *arnq_status_string(arnq_status s) {
  switch (s) {
    case ARNQ_OK: return "ARNQ_OK";
    case ARNQ_ERR_NULL_PTR: return "ARNQ_ERR_NULL_PTR: a required input or a selected output is NULL";
    case ARNQ_ERR_EMPTY: return "ARNQ_ERR_EMPTY: empty tensors are not supported";
    case ARNQ_ERR_SHAPE: return "ARNQ_ERR_SHAPE: unsupported shape (odd n for INT4, n too large, negative size)";
    case ARNQ_ERR_DTYPE: return "ARNQ_ERR_DTYPE: unknown dtype or qdtype";
    case ARNQ_ERR_MASK: return "ARNQ_ERR_MASK: outputMask / smooth-scale combination not allowed";
    case ARNQ_ERR_EPS: return "ARNQ_ERR_EPS: epsilon must be finite and >= 0";
    case ARNQ_ERR_ALIGN: return "ARNQ_ERR_ALIGN: misaligned pointer";
    case ARNQ_ERR_WORKSPACE: return "ARNQ_ERR_WORKSPACE: workspace missing or too small";
    case ARNQ_ERR_CUDA: return "ARNQ_ERR_CUDA: a CUDA call failed";
    case ARNQ_ERR_PLAN: return "ARNQ_ERR_PLAN: the launch plan cannot run this problem";
    case ARNQ_ERR_DEVICE_TIMEOUT: return "ARNQ_ERR_DEVICE_TIMEOUT: a kernel gave up waiting for a copy";
  }
  return "ARNQ: unknown status";
}

arnq_status arnq_selected_outputs(int out_mask, int has_smooth1, int has_smooth2, int *y1_on,
                                  int *y2_on) {
  return selected(out_mask, has_smooth1 != 0, has_smooth2 != 0, y1_on, y2_on);
}

arnq_status arnq_workspace_size(int64_t rows, int64_t n, arnq_dtype dt, arnq_qdtype qdt,
                                int out_mask, int has_smooth1, int has_smooth2, size_t *bytes) {
  if (!bytes) return ARNQ_ERR_NULL_PTR;
  arnq_status st = check_shape(rows, n, dt, qdt, 0.0f);
  if (st != ARNQ_OK) return st;
  st = selected(out_mask, has_smooth1 != 0, has_smooth2 != 0, nullptr, nullptr);
  if (st != ARNQ_OK) return st;
  *bytes = kWorkspaceBytes;
  return ARNQ_OK;
}

arnq_status arnq_run(const void *x1, const void *x2, const void *gamma, const void *beta,
                     const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                     arnq_dtype dt, float eps, int out_mask, arnq_qdtype qdt, void *y1,
                     float *scale1, void *y2, float *scale2, void *x_out, void *workspace,
                     size_t workspace_bytes, void *stream) {
  return run_common(problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, qdt, y1,
                            scale1, y2, scale2, x_out),
                    true, out_mask, workspace, workspace_bytes, stream, nullptr);
}

arnq_status arnq_run_planned(const void *x1, const void *x2, const void *gamma,
                             const void *beta, const void *smooth1, const void *smooth2,
                             int64_t rows, int64_t n, arnq_dtype dt, float eps, int out_mask,
                             arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                             void *x_out, void *workspace, size_t workspace_bytes, void *stream,
                             const arnq_plan *plan) {
  if (!plan) return ARNQ_ERR_NULL_PTR;
  return run_common(problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, qdt, y1,
                            scale1, y2, scale2, x_out),
                    true, out_mask, workspace, workspace_bytes, stream, plan);
}

arnq_status arnq_run_v1(const void *x1, const void *x2, const void *gamma, const void *smooth1,
                        const void *smooth2, int64_t rows, int64_t n, arnq_dtype dt, float eps,
                        arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                        void *x_out, void *workspace, size_t workspace_bytes, void *stream) {
  return arnq_run(x1, x2, gamma, nullptr, smooth1, smooth2, rows, n, dt, eps, ARNQ_MASK_ABSENT,
                  qdt, y1, scale1, y2, scale2, x_out, workspace, workspace_bytes, stream);
}

arnq_status arnq_rms_norm_dynamic_quant(const void *x, const void *gamma, const void *beta,
                                        const void *smooth, int64_t rows, int64_t n,
                                        arnq_dtype dt, float eps, arnq_qdtype qdt, void *y,
                                        float *scale, void *workspace, size_t workspace_bytes,
                                        void *stream) {
  // one output, selected as with the mask absent and only smoothScale1 given
  return run_common(problem(x, nullptr, gamma, beta, smooth, nullptr, rows, n, dt, eps, qdt, y,
                            scale, nullptr, nullptr, nullptr),
                    false, ARNQ_MASK_ABSENT, workspace, workspace_bytes, stream, nullptr);
}

arnq_status arnq_make_plan(const void *x1, const void *x2, const void *gamma, const void *beta,
                           const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                           arnq_dtype dt, int out_mask, arnq_qdtype qdt, const void *y1,
                           const void *y2, const void *x_out, arnq_plan *plan) {
  if (!plan) return ARNQ_ERR_NULL_PTR;
  Problem P = problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, 0.0f, qdt,
                      const_cast<void *>(y1), nullptr, const_cast<void *>(y2), nullptr,
                      const_cast<void *>(x_out));
  arnq_status st = check_shape(rows, n, dt, qdt, 0.0f);
  if (st != ARNQ_OK) return st;
  int on1 = 0, on2 = 0;
  st = selected(out_mask, smooth1 != nullptr, smooth2 != nullptr, &on1, &on2);
  if (st != ARNQ_OK) return st;
  int f = 0;
  if (x2) f |= arnq::F_X2;
  if (beta) f |= arnq::F_BETA;
  if (smooth1) f |= arnq::F_S1;
  if (smooth2) f |= arnq::F_S2;
  if (on1) f |= arnq::F_OUT1;
  if (on2) f |= arnq::F_OUT2;
  if (x2 && x_out) f |= arnq::F_XOUT;
  P.flags = f;
  KernelFn fn = nullptr;
  int smem = 0, seg = 0, units = 0;
  return make_plan(P, plan, &fn, &smem, &seg, &units);
}

}  // extern "C"
