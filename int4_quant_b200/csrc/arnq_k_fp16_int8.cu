// Row-kernel instantiations for fp16 inputs and int8 codes.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int8(KernelFn *t) { fill_quarter<Fp16, false>(t); }
}  // namespace arnq
