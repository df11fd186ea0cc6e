// Row-kernel instantiations for bf16 inputs and int8 codes, one CTA per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int8(KernelFn *t) { fill_quarter<Bf16, false, false>(t); }
}  // namespace arnq
