// Row-kernel instantiations for fp16 inputs and int8 codes, one CTA per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int8(KernelFn *t) { fill_quarter<Fp16, false, false>(t); }
}  // namespace arnq
