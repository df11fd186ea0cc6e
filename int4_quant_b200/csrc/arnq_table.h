// arnq_table.h -- the table of row-kernel instantiations the host dispatches
// into, indexed by output count, add / no-add, load mode, units per thread
// and whether the row is shared by a cluster.  Each (dtype, code type) quarter of the table is
// instantiated in its own translation unit so they compile in parallel.
#pragma once

#include "arnq_kernels.cuh"

namespace arnq {

typedef void (*KernelFn)(KParams);

constexpr int kModes = 3;
constexpr int kUptSlots = 3;   // 16-byte units: 1, 2, 4; element pairs: 1, 4, 8
constexpr int kTableSize = 2 * 2 * kModes * kUptSlots * 2;

inline int upt_slot(int mode, int upt) {
  if (mode == LOAD_SCALAR) return upt == 1 ? 0 : upt == 4 ? 1 : upt == 8 ? 2 : -1;
  return upt == 1 ? 0 : upt == 2 ? 1 : upt == 4 ? 2 : -1;
}

inline int table_index(int nout, bool add, int mode, int slot, bool cl) {
  return ((((nout - 1) * 2 + (add ? 1 : 0)) * kModes + mode) * kUptSlots + slot) * 2 +
         (cl ? 1 : 0);
}

// Four 16-byte units per thread with one output use the 96-register entry
// point (five CTAs per SM); every other variant the launch-bounds one.
template <class T, bool I4, int MODE, int NOUT, bool ADD, bool CL>
constexpr KernelFn upt4_kernel() {
  if constexpr (NOUT == 1) return rows_kernel_r96<T, I4, MODE, 4, NOUT, ADD, CL>;
  else return rows_kernel<T, I4, MODE, 4, NOUT, ADD, CL>;
}

template <class T, bool I4, int NOUT, bool ADD, bool CL>
void fill_na(KernelFn *t) {
  t[table_index(NOUT, ADD, LOAD_VEC, 0, CL)] = rows_kernel<T, I4, LOAD_VEC, 1, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_VEC, 1, CL)] = rows_kernel<T, I4, LOAD_VEC, 2, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_VEC, 2, CL)] = upt4_kernel<T, I4, LOAD_VEC, NOUT, ADD, CL>();
  t[table_index(NOUT, ADD, LOAD_STAGED, 0, CL)] =
      rows_kernel<T, I4, LOAD_STAGED, 1, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_STAGED, 1, CL)] =
      rows_kernel<T, I4, LOAD_STAGED, 2, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_STAGED, 2, CL)] = upt4_kernel<T, I4, LOAD_STAGED, NOUT, ADD, CL>();
  t[table_index(NOUT, ADD, LOAD_SCALAR, 0, CL)] =
      rows_kernel<T, I4, LOAD_SCALAR, 1, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_SCALAR, 1, CL)] =
      rows_kernel<T, I4, LOAD_SCALAR, 4, NOUT, ADD, CL>;
  t[table_index(NOUT, ADD, LOAD_SCALAR, 2, CL)] =
      rows_kernel<T, I4, LOAD_SCALAR, 8, NOUT, ADD, CL>;
}

// One CTA per row (CL = false) or a cluster per row (CL = true).
template <class T, bool I4, bool CL>
void fill_quarter(KernelFn *t) {
  fill_na<T, I4, 1, false, CL>(t);
  fill_na<T, I4, 1, true, CL>(t);
  fill_na<T, I4, 2, false, CL>(t);
  fill_na<T, I4, 2, true, CL>(t);
}

// Defined one per translation unit (arnq_k_<dtype>_<codes>[_cl].cu).
void fill_table_bf16_int8(KernelFn *t);
void fill_table_bf16_int4(KernelFn *t);
void fill_table_fp16_int8(KernelFn *t);
void fill_table_fp16_int4(KernelFn *t);
void fill_table_bf16_int8_cl(KernelFn *t);
void fill_table_bf16_int4_cl(KernelFn *t);
void fill_table_fp16_int8_cl(KernelFn *t);
void fill_table_fp16_int4_cl(KernelFn *t);

}  // namespace arnq
