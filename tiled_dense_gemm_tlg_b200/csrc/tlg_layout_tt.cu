// Kernel instantiations for one operand layout: A stored transposed, B stored transposed.
#include "tlg_variants.cuh"

namespace tlg {

const LayoutTables kLayoutTT = {TLG_LAYOUT(true, true), TLG_LAYOUT_PLAIN(true, true)};

TLG_DEFINE_ERROR_WORD_READER(error_word_tt)

}  // namespace tlg
