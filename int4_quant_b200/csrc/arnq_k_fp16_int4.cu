// Row-kernel instantiations for fp16 inputs and int4 codes, one CTA per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int4(KernelFn *t) { fill_quarter<Fp16, true, false>(t); }
}  // namespace arnq
