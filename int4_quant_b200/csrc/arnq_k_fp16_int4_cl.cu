// Row-kernel instantiations for fp16 inputs and int4 codes, a cluster per row.
#include "arnq_table.h"

namespace arnq {
void fill_table_fp16_int4_cl(KernelFn *t) { fill_quarter<Fp16, true, true>(t); }
}  // namespace arnq
