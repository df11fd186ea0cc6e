// Row-kernel instantiations for bf16 inputs and int8 codes.
#include "arnq_table.h"

namespace arnq {
void fill_table_bf16_int8(KernelFn *t) { fill_quarter<Bf16, false>(t); }
}  // namespace arnq
