// Row-kernel instantiations for bf16 inputs and int4 codes, a cluster per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int4_cl(KernelFn *t) { fill_quarter<Bf16, true, true>(t); }
}  // namespace arnq
