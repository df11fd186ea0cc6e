// Row-kernel instantiations for fp16 inputs and int8 codes, a cluster per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int8_cl(KernelFn *t) { fill_quarter<Fp16, false, true>(t); }
}  // namespace arnq
