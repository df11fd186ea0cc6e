// Row-kernel instantiations for fp16 inputs and int8 codes, one CTA per row, and the settle kernels.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int8(KernelFn *t) { fill_quarter<Fp16, false, false>(t); }
void fill_settle_fp16_int8(SettleFn *t) { fill_settle<Fp16, false>(t); }
}  // namespace arnq
