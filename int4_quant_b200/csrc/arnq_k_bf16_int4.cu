// Row-kernel instantiations for bf16 inputs and int4 codes, one CTA per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int4(KernelFn *t) { fill_quarter<Bf16, true, false>(t); }
}  // namespace arnq
