// Kernel instantiations for one operand layout: A stored transposed, B as stored.
#include "tlg_variants.cuh"

namespace tlg {

const LayoutTables kLayoutTN = {TLG_LAYOUT(true, false), TLG_LAYOUT_PLAIN(true, false)};

TLG_DEFINE_ERROR_WORD_READER(error_word_tn)

}  // namespace tlg
