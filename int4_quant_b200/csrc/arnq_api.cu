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
#include "arnq_table.h"

namespace {

using arnq::KParams;
using arnq::KernelFn;

// workspace: the status block only (the row records live in shared memory),
// whatever the problem
size_t workspace_bytes_for() { return static_cast<size_t>(arnq::kStatusBytes); }
constexpr int kMaxStages = arnq::kMaxStagesDev;
constexpr int kMaxCluster = 16;

// ---------------------------------------------------------------- kernel table

struct KernelTable {
  KernelFn fn[2][2][arnq::kTableSize];  // [dtype][qdtype][...]
  KernelTable() {
    std::memset(fn, 0, sizeof fn);
    arnq::fill_table_bf16_int8(fn[0][0]);
    arnq::fill_table_bf16_int4(fn[0][1]);
    arnq::fill_table_fp16_int8(fn[1][0]);
    arnq::fill_table_fp16_int4(fn[1][1]);
    arnq::fill_table_bf16_int8_cl(fn[0][0]);
    arnq::fill_table_bf16_int4_cl(fn[0][1]);
    arnq::fill_table_fp16_int8_cl(fn[1][0]);
    arnq::fill_table_fp16_int4_cl(fn[1][1]);
  }
};

const KernelTable &kernel_table() {
  static const KernelTable table;
  return table;
}

// The eight-codes-per-word INT4 container has the byte layout of packed INT4
// on a little-endian device (code 8w + k in bits 4k..4k+3 of word w is the
// low nibble of byte 4w + k/2 for even k, the high nibble for odd k): the
// INT4 kernels write it.
KernelFn lookup(int dt, int qdt, int nout, bool add, int mode, int upt, int cluster) {
  if (qdt == ARNQ_INT4_INT32) qdt = ARNQ_INT4;
  const KernelTable &table = kernel_table();
  const int s = arnq::upt_slot(mode, upt);
  if (s < 0 || nout < 1 || nout > 2) return nullptr;
  return table.fn[dt][qdt][arnq::table_index(nout, add, mode, s, cluster > 1)];
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
  bool add;       // x = x1 + x2 (else x = x1: the no-add operator)
  bool on1, on2;  // selected outputs
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
  if (qdt != ARNQ_INT8 && qdt != ARNQ_INT4 && qdt != ARNQ_INT4_INT32) return ARNQ_ERR_DTYPE;
  if (rows < 0 || n < 0) return ARNQ_ERR_SHAPE;
  if (rows > INT32_MAX) return ARNQ_ERR_SHAPE;  // row indices are 32-bit in the kernels' lists
  if (rows == 0 || n == 0) return ARNQ_ERR_EMPTY;
  if (n > ARNQ_MAX_N) return ARNQ_ERR_SHAPE;
  if (qdt == ARNQ_INT4 && (n % 2) != 0) return ARNQ_ERR_SHAPE;
  if (qdt == ARNQ_INT4_INT32 && (n % 8) != 0) return ARNQ_ERR_SHAPE;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return ARNQ_ERR_EPS;
  return ARNQ_OK;
}

// Decides the selected outputs and drops the pointers of the others.
arnq_status select_outputs(Problem &P, int out_mask) {
  int on1 = 0, on2 = 0;
  arnq_status st = selected(out_mask, P.s1 != nullptr, P.s2 != nullptr, &on1, &on2);
  if (st != ARNQ_OK) return st;
  P.on1 = on1 != 0;
  P.on2 = on2 != 0;
  if (!P.on1) { P.y1 = nullptr; P.scale1 = nullptr; }
  if (!P.on2) { P.y2 = nullptr; P.scale2 = nullptr; }
  if (!P.add) { P.x2 = nullptr; P.x_out = nullptr; }
  return ARNQ_OK;
}

arnq_status validate(Problem &P, int out_mask, const void *workspace, size_t workspace_bytes) {
  arnq_status st = check_shape(P.rows, P.n, P.dt, P.qdt, P.eps);
  if (st != ARNQ_OK) return st;
  st = select_outputs(P, out_mask);
  if (st != ARNQ_OK) return st;
  if (!P.x1 || (P.add && !P.x2) || !P.gamma) return ARNQ_ERR_NULL_PTR;
  if (P.on1 && (!P.y1 || !P.scale1)) return ARNQ_ERR_NULL_PTR;
  if (P.on2 && (!P.y2 || !P.scale2)) return ARNQ_ERR_NULL_PTR;
  const void *h16[] = {P.x1, P.x2, P.gamma, P.beta, P.s1, P.s2, P.x_out};
  for (const void *q : h16)
    if (q && !aligned(q, 2)) return ARNQ_ERR_ALIGN;
  if ((P.on1 && !aligned(P.scale1, 4)) || (P.on2 && !aligned(P.scale2, 4))) return ARNQ_ERR_ALIGN;
  if (P.qdt == ARNQ_INT4_INT32 && ((P.on1 && !aligned(P.y1, 4)) || (P.on2 && !aligned(P.y2, 4))))
    return ARNQ_ERR_ALIGN;
  if (!workspace || workspace_bytes < workspace_bytes_for()) return ARNQ_ERR_WORKSPACE;
  if (!aligned(workspace, 8)) return ARNQ_ERR_ALIGN;
  return ARNQ_OK;
}

// ---------------------------------------------------------------- planning

int round_up(int v, int m) { return (v + m - 1) / m * m; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// 16-byte units need every 16-bit tensor 16-byte aligned with n % 8 == 0 (so
// each row starts aligned), and the code outputs aligned to their 8 (INT8) or
// 4 (INT4) bytes per unit.
bool vector_ok(const Problem &P) {
  if (P.n % 8 != 0) return false;
  const void *v16[] = {P.x1, P.x2, P.gamma, P.beta, P.s1, P.s2, P.x_out};
  for (const void *q : v16)
    if (q && !aligned(q, 16)) return false;
  const uintptr_t ya = (P.qdt == ARNQ_INT8) ? 8 : 4;
  if (P.on1 && !aligned(P.y1, ya)) return false;
  if (P.on2 && !aligned(P.y2, ya)) return false;
  return true;
}

struct Launch {
  KernelFn fn;
  int smem, seg, units;
  int tail_rows, trec_bytes;  // row records per CTA (cluster) and their bytes
};

int upt_candidate(int mode, int i) {
  static const int vec[3] = {1, 2, 4}, sca[3] = {1, 4, 8};
  return mode == arnq::LOAD_SCALAR ? sca[i] : vec[i];
}

// Shared memory of one CTA: the exchange slots, `tail_rows` row records,
// B_k of 16-byte units, then (staged) the input ring.
int smem_bytes(int mode, int upt, int cl, int threads, int nout, int stages, int stage_bytes,
               int tail_rows, int trec_bytes) {
  const arnq::Layout lay = arnq::make_layout(
      cl * (threads / 32), nout, stages, tail_rows, trec_bytes,
      arnq::bsm_bytes_for(mode != arnq::LOAD_SCALAR, nout, upt, threads));
  return lay.ring + stages * stage_bytes;
}

// CTAs of `fn` resident per SM (from its actual register count and the smem).
arnq_status occupancy(KernelFn fn, int threads, int smem, int *per_sm) {
  *per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, fn, threads, smem) != cudaSuccess)
    return ARNQ_ERR_CUDA;
  return ARNQ_OK;
}

// Requested plan fields that no plan can take (checked before any device query).
arnq_status check_plan_fields(const arnq_plan &q) {
  if (q.wait_limit_us < 0 || q.test_hold_bytes < 0 || q.test_hold_bytes > 65536 || q.grid < 0 ||
      q.ctas_per_sm < 0 || q.early_params < 0 || q.early_params > 1 || q.stages < 0 ||
      q.threads < 0 ||
      q.units < 0 || q.cluster < 0)
    return ARNQ_ERR_PLAN;
  return ARNQ_OK;
}

arnq_status make_plan(const Problem &P, arnq_plan *pl, Launch *L) {
  arnq_status st = check_plan_fields(*pl);
  if (st != ARNQ_OK) return st;
  DeviceInfo di;
  int dev = 0;
  st = device_info(&di, &dev);
  if (st != ARNQ_OK) return st;
  const bool vec = vector_ok(P);
  const int nout = (P.on1 ? 1 : 0) + (P.on2 ? 1 : 0);
  if (pl->kernel == ARNQ_KERNEL_AUTO) pl->kernel = vec ? ARNQ_KERNEL_STAGED : ARNQ_KERNEL_DIRECT;
  if (pl->kernel == ARNQ_KERNEL_STAGED && !vec) return ARNQ_ERR_PLAN;
  if (pl->kernel != ARNQ_KERNEL_DIRECT && pl->kernel != ARNQ_KERNEL_STAGED) return ARNQ_ERR_PLAN;
  const int mode = pl->kernel == ARNQ_KERNEL_STAGED ? arnq::LOAD_STAGED
                   : vec                            ? arnq::LOAD_VEC
                                                    : arnq::LOAD_SCALAR;
  pl->vector = (mode != arnq::LOAD_SCALAR) ? 1 : 0;
  const int U = (mode == arnq::LOAD_SCALAR) ? 2 : 8;
  const int units = static_cast<int>(ceil_div(P.n, U));
  const int nin = P.add ? 2 : 1;
  // the most units one CTA can hold (units per thread times the threads allowed,
  // for the requested units per thread or the best of them)
  int max_seg = 0;
  for (int i = 0; i < 3; ++i) {
    const int c = upt_candidate(mode, i);
    if (pl->units != 0 && c != pl->units) continue;
    const int m = c * arnq::max_threads_for(mode, c, nout);
    if (m > max_seg) max_seg = m;
  }
  if (max_seg == 0) return ARNQ_ERR_PLAN;

  // cluster: enough CTAs per row that one CTA's slice fits in registers (and,
  // staged, one stage of it and its B_k in shared memory).  No more: with
  // fewer rows than SMs, a cluster spreading each row over more SMs measured
  // slower than one CTA per row with more threads (B200, device time per
  // call, L2-cold: 64 x 1024 4.4 us with one 128-thread CTA per row, 8.6 us
  // as 2-CTA clusters; 128 x 16384 9.7 vs 12.8 us; 1 x 16384 7.4 vs 10.1 us
  // as a 16-CTA cluster)
  if (pl->cluster == 0) {
    int cl = 1;
    auto too_big = [&](int c) {
      const int64_t seg = ceil_div(units, c);
      if (seg > max_seg) return true;
      return mode == arnq::LOAD_STAGED &&
             nin * seg * 16 + nout * seg * 32 + 8192 > di.smem_per_block_optin;
    };
    while (cl < kMaxCluster && too_big(cl)) cl *= 2;
    pl->cluster = cl;
  }
  const int cl = pl->cluster;
  if (cl != 1 && cl != 2 && cl != 4 && cl != 8 && cl != 16) return ARNQ_ERR_PLAN;
  const int seg = static_cast<int>(ceil_div(units, cl));
  if (seg > max_seg) return ARNQ_ERR_PLAN;
  const int stage_bytes = nin * seg * 16;
  const int trec = arnq::tail_rec_bytes(arnq::tie_cap(static_cast<int>(P.n), nout));

  // units per thread: of the variants whose threads hold a slice, the one with
  // the most CTAs (rows in flight) per SM, then the most units per thread
  // (fewer threads share a row: cheaper reductions); measured best on
  // 4096..16384-column rows.  With fewer rows than SMs (each row has an SM
  // to itself, latency rules): the fewest units per thread, i.e. the most
  // threads on a row (64 x 1024: 4.4 us with 1 unit per thread, 5.8 us with 4)
  if (pl->units == 0 && P.rows < di.sms) {
    for (int i = 0; i < 3 && pl->units == 0; ++i) {
      const int c = upt_candidate(mode, i);
      const int t = round_up(static_cast<int>(ceil_div(seg, c)), 32);
      if (t <= arnq::max_threads_for(mode, c, nout) && lookup(P.dt, P.qdt, nout, P.add, mode, c, cl))
        pl->units = c;
    }
  }
  if (pl->units == 0) {
    int best = 0, best_ctas = -1;
    for (int i = 0; i < 3; ++i) {
      const int c = upt_candidate(mode, i);
      const int t = round_up(static_cast<int>(ceil_div(seg, c)), 32);
      if (t > arnq::max_threads_for(mode, c, nout)) continue;
      if (ceil_div(seg, c) < 32 && best != 0) continue;  // no more than a warp's worth idle
      KernelFn f = lookup(P.dt, P.qdt, nout, P.add, mode, c, cl);
      if (!f) continue;
      const int sm = smem_bytes(mode, c, cl, t, nout, mode == arnq::LOAD_STAGED ? 1 : 0,
                                stage_bytes, 1, trec);
      if (sm > di.smem_per_block_optin) continue;
      st = prepare_kernel(f, dev, sm);
      if (st != ARNQ_OK) return st;
      int per_sm = 0;
      st = occupancy(f, t, sm, &per_sm);
      if (st != ARNQ_OK) return st;
      if (per_sm < 1) continue;
      if (per_sm > best_ctas || (per_sm == best_ctas && c > best)) {
        best = c;
        best_ctas = per_sm;
      }
    }
    if (best == 0) return ARNQ_ERR_PLAN;
    pl->units = best;
  }
  if (arnq::upt_slot(mode, pl->units) < 0) return ARNQ_ERR_PLAN;
  const int tmax = arnq::max_threads_for(mode, pl->units, nout);
  if (pl->threads == 0) {
    pl->threads = round_up(static_cast<int>(ceil_div(seg, pl->units)), 32);
    if (pl->threads < 32) pl->threads = 32;
  }
  if (pl->threads % 32 != 0 || pl->threads > tmax ||
      static_cast<int64_t>(pl->threads) * pl->units < seg)
    return ARNQ_ERR_PLAN;

  KernelFn fn = lookup(P.dt, P.qdt, nout, P.add, mode, pl->units, cl);
  if (!fn) return ARNQ_ERR_PLAN;
  const int upt = pl->units;

  // Resident clusters (CTAs when cl == 1), grid and records per cluster for a
  // ring depth `stages`.  A cluster keeps one record per row it processes in
  // its first CTA's shared memory, so shared memory grows with the rows per
  // cluster.  Every resident slot gets a cluster (more rows in flight beat
  // equal row counts: on 8192 x 4096, 740 CTAs took 44.3 us a call, the 683
  // that give every CTA 12 rows 46.2 us), no more clusters than rows; while
  // the records do not fit, fewer clusters per SM with more rows each; when
  // not even one cluster can hold its rows' records, a grid run in waves with
  // fewer rows per cluster.  A requested grid is kept.
  struct Eval {
    int per_sm = 0, smem = 0, tail_rows = 0;
    int64_t nclusters = 0;
  };
  const int spare = 0;
  // clusters resident at once with `sm` bytes of shared memory per CTA
  auto resident = [&](int sm, int *per_sm, int64_t *slots) -> arnq_status {
    *per_sm = 0;
    *slots = 0;
    arnq_status s2 = prepare_kernel(fn, dev, sm);
    if (s2 != ARNQ_OK) return s2;
    if (cl > 1) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cl;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cl * 1024, 1, 1);
      cfg.blockDim = dim3(pl->threads, 1, 1);
      cfg.dynamicSmemBytes = sm;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, fn, &cfg) != cudaSuccess) return ARNQ_ERR_CUDA;
      if (nc < 1) return ARNQ_OK;
      int64_t want =
          pl->ctas_per_sm != 0 ? static_cast<int64_t>(pl->ctas_per_sm) * di.sms / cl : nc;
      if (want < 1) want = 1;
      *slots = want < nc ? want : nc;
      *per_sm = static_cast<int>(ceil_div(*slots * cl, di.sms));
      return ARNQ_OK;
    }
    int ps = 0;
    s2 = occupancy(fn, pl->threads, sm, &ps);
    if (s2 != ARNQ_OK) return s2;
    if (ps < 1) return ARNQ_OK;
    if (pl->ctas_per_sm != 0 && pl->ctas_per_sm < ps) ps = pl->ctas_per_sm;
    *per_sm = ps;
    *slots = static_cast<int64_t>(ps) * di.sms;
    return ARNQ_OK;
  };
  // shared memory of a CTA holding `nrec` records; false if beyond the limit
  auto smem_for = [&](int stages, int64_t nrec, int *sm) -> bool {
    if (nrec * static_cast<int64_t>(trec) > di.smem_per_block_optin) return false;
    *sm = smem_bytes(mode, upt, cl, pl->threads, nout, stages, stage_bytes,
                     static_cast<int>(nrec), trec);
    return *sm <= di.smem_per_block_optin;
  };
  auto evaluate = [&](int stages, Eval *e) -> arnq_status {
    *e = Eval();
    int sm = 0, per_sm = 0;
    int64_t slots = 0;
    if (!smem_for(stages, 1 + spare, &sm)) return ARNQ_OK;
    arnq_status s2 = resident(sm, &per_sm, &slots);
    if (s2 != ARNQ_OK) return s2;
    if (slots < 1) return ARNQ_OK;
    const bool fixed = pl->grid != 0;
    if (fixed && pl->grid % cl != 0) return ARNQ_ERR_PLAN;
    int64_t ncl = fixed ? pl->grid / cl : (P.rows < slots ? P.rows : slots);
    for (int iter = 0; iter < 32; ++iter) {  // ncl only decreases
      const int64_t nrec = ceil_div(P.rows, ncl) + spare;
      int fps = 0;
      int64_t fit = 0;
      if (smem_for(stages, nrec, &sm)) {
        s2 = resident(sm, &fps, &fit);
        if (s2 != ARNQ_OK) return s2;
      }
      if (fit >= 1 && (fixed || fit >= ncl)) {
        e->per_sm = fps;
        e->nclusters = ncl;
        e->tail_rows = static_cast<int>(nrec);
        e->smem = sm;
        return ARNQ_OK;
      }
      if (fixed || fit < 1) break;
      ncl = fit;  // fewer clusters, more rows (records) each
    }
    if (fixed) return ARNQ_OK;
    // not even one resident cluster holds its rows' records: fewer rows per
    // cluster, a grid run in waves
    int64_t rows_per = ceil_div(P.rows, slots);
    while (true) {
      int fps = 0;
      int64_t fit = 0;
      if (smem_for(stages, rows_per + spare, &sm)) {
        s2 = resident(sm, &fps, &fit);
        if (s2 != ARNQ_OK) return s2;
      }
      if (fit >= 1) {
        e->per_sm = fps;
        e->nclusters = ceil_div(P.rows, rows_per);
        e->tail_rows = static_cast<int>(rows_per + spare);
        e->smem = sm;
        return ARNQ_OK;
      }
      if (rows_per == 1) return ARNQ_OK;
      rows_per = ceil_div(rows_per, 2);
    }
  };

  Eval best;
  if (mode == arnq::LOAD_STAGED) {
    // ring depth: the one (of 1 and 2) that keeps the most CTAs, i.e. rows in
    // flight, on an SM; two on a tie (measured on 4096-column rows: five CTAs
    // with one stage beat four with two)
    if (pl->stages != 0 && (pl->stages < 1 || pl->stages > kMaxStages)) return ARNQ_ERR_PLAN;
    int best_s = 0;
    for (int s = 1; s <= kMaxStages; ++s) {
      if (pl->stages != 0 ? s != pl->stages : s > 2) continue;
      Eval e;
      st = evaluate(s, &e);
      if (st != ARNQ_OK) return st;
      if (e.per_sm > 0 && e.per_sm >= best.per_sm) {
        best = e;
        best_s = s;
      }
    }
    if (best_s == 0) return ARNQ_ERR_PLAN;
    pl->stages = best_s;
  } else {
    pl->stages = 0;
    st = evaluate(0, &best);
    if (st != ARNQ_OK) return st;
    if (best.per_sm == 0) return ARNQ_ERR_PLAN;
  }
  st = prepare_kernel(fn, dev, best.smem);
  if (st != ARNQ_OK) return st;
  pl->ctas_per_sm = best.per_sm;
  const int64_t nclusters = best.nclusters;
  const int smem = best.smem;
  pl->grid = static_cast<int32_t>(nclusters * cl);
  L->tail_rows = best.tail_rows;
  L->trec_bytes = trec;
  L->fn = fn;
  L->smem = smem;
  L->seg = seg;
  L->units = units;
  return ARNQ_OK;
}

// Plans depend on the device, the shape, the dtypes, the outputs, whether the
// 16-byte path applies, whether xOut is written and the requested plan
// fields, not on the pointers:
// cached per key, so that repeated calls skip the occupancy queries.
struct PlanKey {
  int dev;
  int64_t rows, n;
  int dt, qdt, nout, add, vec, beta, xout;
  arnq_plan req;
};
struct PlanEntry {
  bool used;
  PlanKey key;
  arnq_plan plan;
  Launch L;
};
constexpr int kPlanCache = 64;
PlanEntry g_plans[kPlanCache];
int g_plan_next = 0;

bool same_key(const PlanKey &a, const PlanKey &b) { return std::memcmp(&a, &b, sizeof a) == 0; }

// The last plan this thread used: a call with the same key (a decode loop
// calls with one shape over and over) takes it without the lock.  Entries are
// never invalidated: a plan depends only on its key.
struct LastPlan {
  bool used = false;
  PlanKey key;
  arnq_plan plan;
  Launch L;
};
thread_local LastPlan t_last;

arnq_status make_plan_cached(const Problem &P, arnq_plan *pl, Launch *L) {
  PlanKey key;
  std::memset(&key, 0, sizeof key);  // padding too: keys compare bytewise
  if (cudaGetDevice(&key.dev) != cudaSuccess) return ARNQ_ERR_CUDA;
  key.rows = P.rows;
  key.n = P.n;
  key.dt = P.dt;
  key.qdt = P.qdt;
  key.nout = (P.on1 ? 1 : 0) + (P.on2 ? 1 : 0);
  key.add = P.add ? 1 : 0;
  key.vec = vector_ok(P) ? 1 : 0;
  key.beta = P.beta ? 1 : 0;
  key.xout = P.x_out ? 1 : 0;  // where the settling reads x back from
  key.req = *pl;
  if (t_last.used && same_key(t_last.key, key)) {
    *pl = t_last.plan;
    *L = t_last.L;
    return ARNQ_OK;
  }
  auto remember = [&]() {
    t_last.used = true;
    t_last.key = key;
    t_last.plan = *pl;
    t_last.L = *L;
  };
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < kPlanCache; ++i)
      if (g_plans[i].used && same_key(g_plans[i].key, key)) {
        *pl = g_plans[i].plan;
        *L = g_plans[i].L;
        remember();
        return ARNQ_OK;
      }
  }
  arnq_status st = make_plan(P, pl, L);
  if (st != ARNQ_OK) return st;
  remember();
  std::lock_guard<std::mutex> lock(g_mu);
  PlanEntry &e = g_plans[g_plan_next];
  g_plan_next = (g_plan_next + 1) % kPlanCache;
  e.used = true;
  e.key = key;
  e.plan = *pl;
  e.L = *L;
  return ARNQ_OK;
}

arnq_status launch(const Problem &P, arnq_plan plan, void *workspace, cudaStream_t stream) {
  Launch L;
  arnq_status st = make_plan_cached(P, &plan, &L);
  if (st != ARNQ_OK) return st;
  KParams k;
  std::memset(&k, 0, sizeof k);
  k.x1 = static_cast<const uint16_t *>(P.x1);
  k.x2 = static_cast<const uint16_t *>(P.x2);
  k.gamma = static_cast<const uint16_t *>(P.gamma);
  k.beta = static_cast<const uint16_t *>(P.beta);
  // output slots: the selected outputs in order, each with its own smooth scale
  int slot = 0;
  if (P.on1) {
    k.smooth[slot] = static_cast<const uint16_t *>(P.s1);
    k.y[slot] = static_cast<uint8_t *>(P.y1);
    k.scale[slot] = P.scale1;
    ++slot;
  }
  if (P.on2) {
    k.smooth[slot] = static_cast<const uint16_t *>(P.s2);
    k.y[slot] = static_cast<uint8_t *>(P.y2);
    k.scale[slot] = P.scale2;
    ++slot;
  }
  k.x_out = static_cast<uint16_t *>(P.x_out);
  k.status = static_cast<int32_t *>(workspace);
  k.tie_cap = arnq::tie_cap(static_cast<int>(P.n), (P.on1 ? 1 : 0) + (P.on2 ? 1 : 0));
  k.tail_rows = L.tail_rows;
  k.trec_bytes = L.trec_bytes;
  k.rows = P.rows;
  k.n = static_cast<int32_t>(P.n);
  k.units = L.units;
  k.seg_units = L.seg;
  k.flags = (P.beta ? arnq::F_BETA : 0) | (P.add && P.x_out ? arnq::F_XOUT : 0) |
            (plan.early_params ? arnq::F_EARLY : 0);
  k.stages = plan.stages;
  k.eps = P.eps;
  k.inv_n = 1.0 / static_cast<double>(P.n);
  k.wait_limit_ns = plan.wait_limit_us > 0
                        ? static_cast<uint64_t>(plan.wait_limit_us) * 1000ull
                        : static_cast<uint64_t>(arnq::kWaitLimitNs);
  k.test_hold_tx = plan.kernel == ARNQ_KERNEL_STAGED && plan.test_hold_bytes > 0
                       ? static_cast<uint32_t>(plan.test_hold_bytes)
                       : 0u;

  // The row kernel is a programmatic dependent of whatever precedes it on the
  // stream: its CTAs may become resident while that work finishes, and wait
  // (griddepcontrol.wait) for it before touching memory.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (plan.cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = plan.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, L.fn, k) != cudaSuccess) return ARNQ_ERR_CUDA;
  return ARNQ_OK;
}

Problem problem(const void *x1, const void *x2, const void *gamma, const void *beta,
                const void *s1, const void *s2, int64_t rows, int64_t n, arnq_dtype dt,
                float eps, arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                void *x_out, bool add) {
  Problem P;
  P.x1 = x1; P.x2 = x2; P.gamma = gamma; P.beta = beta; P.s1 = s1; P.s2 = s2;
  P.y1 = y1; P.y2 = y2; P.x_out = x_out; P.scale1 = scale1; P.scale2 = scale2;
  P.rows = rows; P.n = n; P.dt = static_cast<int>(dt); P.qdt = static_cast<int>(qdt);
  P.eps = eps; P.add = add; P.on1 = P.on2 = false;
  return P;
}

// ---------------------------------------------------------------- static scratch

// The no-allocation entry point's scratch: one array per device, in the
// library's own device memory (zero when the library's device code is loaded).
// Host code cannot use the symbol as a device address: the address is looked
// up on every call, with the current device, so that it is never stale (a
// device reset between calls reloads the module at another address).
static __device__ __align__(256) unsigned char g_static_scratch[ARNQ_STATIC_SCRATCH_BYTES];

arnq_status static_scratch(void **out) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return ARNQ_ERR_CUDA;
  *out = p;
  return ARNQ_OK;
}

arnq_status run_common(Problem P, int out_mask, void *workspace, size_t workspace_bytes,
                       void *stream, const arnq_plan *plan) {
  arnq_status st = validate(P, out_mask, workspace, workspace_bytes);
  if (st != ARNQ_OK) return st;
  arnq_plan pl;
  std::memset(&pl, 0, sizeof pl);
  if (plan) pl = *plan;
  st = check_plan_fields(pl);
  if (st != ARNQ_OK) return st;
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
    case ARNQ_ERR_SHAPE:
      return "ARNQ_ERR_SHAPE: unsupported shape (n not a multiple of 2 for INT4 or 8 for "
             "INT4_INT32, n too large, negative size)";
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
  int on1 = 0, on2 = 0;
  st = selected(out_mask, has_smooth1 != 0, has_smooth2 != 0, &on1, &on2);
  if (st != ARNQ_OK) return st;
  *bytes = workspace_bytes_for();
  return ARNQ_OK;
}

arnq_status arnq_run(const void *x1, const void *x2, const void *gamma, const void *beta,
                     const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                     arnq_dtype dt, float eps, int out_mask, arnq_qdtype qdt, void *y1,
                     float *scale1, void *y2, float *scale2, void *x_out, void *workspace,
                     size_t workspace_bytes, void *stream) {
  return run_common(problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, qdt, y1,
                            scale1, y2, scale2, x_out, true),
                    out_mask, workspace, workspace_bytes, stream, nullptr);
}

arnq_status arnq_run_planned(const void *x1, const void *x2, const void *gamma,
                             const void *beta, const void *smooth1, const void *smooth2,
                             int64_t rows, int64_t n, arnq_dtype dt, float eps, int out_mask,
                             arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                             void *x_out, void *workspace, size_t workspace_bytes, void *stream,
                             const arnq_plan *plan) {
  if (!plan) return ARNQ_ERR_NULL_PTR;
  return run_common(problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, qdt, y1,
                            scale1, y2, scale2, x_out, true),
                    out_mask, workspace, workspace_bytes, stream, plan);
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
                            scale, nullptr, nullptr, nullptr, false),
                    ARNQ_MASK_ABSENT, workspace, workspace_bytes, stream, nullptr);
}

arnq_status arnq_make_plan(const void *x1, const void *x2, const void *gamma, const void *beta,
                           const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                           arnq_dtype dt, int out_mask, arnq_qdtype qdt, const void *y1,
                           const void *y2, const void *x_out, arnq_plan *plan) {
  if (!plan) return ARNQ_ERR_NULL_PTR;
  Problem P = problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, 0.0f, qdt,
                      const_cast<void *>(y1), nullptr, const_cast<void *>(y2), nullptr,
                      const_cast<void *>(x_out), x2 != nullptr);
  arnq_status st = check_shape(rows, n, dt, qdt, 0.0f);
  if (st != ARNQ_OK) return st;
  st = select_outputs(P, out_mask);
  if (st != ARNQ_OK) return st;
  Launch L;
  return make_plan(P, plan, &L);
}

arnq_status arnq_run_static_scratch(const void *x1, const void *x2, const void *gamma,
                                    const void *beta, const void *smooth1, const void *smooth2,
                                    int64_t rows, int64_t n, arnq_dtype dt, float eps,
                                    int out_mask, arnq_qdtype qdt, void *y1, float *scale1,
                                    void *y2, float *scale2, void *x_out, void *stream) {
  Problem P = problem(x1, x2, gamma, beta, smooth1, smooth2, rows, n, dt, eps, qdt, y1, scale1, y2,
                      scale2, x_out, true);
  // the host-side checks first: a rejected call touches no device
  arnq_status st = check_shape(P.rows, P.n, P.dt, P.qdt, P.eps);
  if (st != ARNQ_OK) return st;
  size_t need = 0;
  st = arnq_workspace_size(rows, n, dt, qdt, out_mask, smooth1 != nullptr, smooth2 != nullptr,
                           &need);
  if (st != ARNQ_OK) return st;
  if (need > ARNQ_STATIC_SCRATCH_BYTES) return ARNQ_ERR_WORKSPACE;
  {
    // every other argument check, with an aligned stand-in for the scratch
    // address (validate only inspects the pointer's value)
    Problem Q = P;
    st = validate(Q, out_mask, reinterpret_cast<void *>(static_cast<uintptr_t>(256)),
                  ARNQ_STATIC_SCRATCH_BYTES);
    if (st != ARNQ_OK) return st;
  }
  void *scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != ARNQ_OK) return st;
  // the status block must start at zero (the kernel writes it only on error)
  if (cudaMemsetAsync(scratch, 0, arnq::kStatusBytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return ARNQ_ERR_CUDA;
  return run_common(P, out_mask, scratch, ARNQ_STATIC_SCRATCH_BYTES, stream, nullptr);
}

}  // extern "C"
