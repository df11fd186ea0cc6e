// Row-kernel instantiations for bf16 inputs and int8 codes, one CTA per row, and the settle kernels.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int8(KernelFn *t) { fill_quarter<Bf16, false, false>(t); }
void fill_settle_bf16_int8(SettleFn *t) { fill_settle<Bf16, false>(t); }
}  // namespace arnq
