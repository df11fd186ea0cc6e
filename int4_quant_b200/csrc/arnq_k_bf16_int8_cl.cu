// Row-kernel instantiations for bf16 inputs and int8 codes, a cluster per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int8_cl(KernelFn *t) { fill_quarter<Bf16, false, true>(t); }
}  // namespace arnq
