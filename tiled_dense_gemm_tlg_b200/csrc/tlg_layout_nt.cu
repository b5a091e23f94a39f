// Kernel instantiations for one operand layout: A as stored, B stored transposed.
#include "tlg_variants.cuh"

namespace tlg {

const LayoutTables kLayoutNT = {TLG_LAYOUT(false, true), TLG_LAYOUT_PLAIN(false, true)};

TLG_DEFINE_ERROR_WORD_READER(error_word_nt)

}  // namespace tlg
