// Kernel instantiations for one operand layout: A as stored, B as stored.
#include "tlg_variants.cuh"

namespace tlg {

const LayoutTables kLayoutNN = {TLG_LAYOUT_NN, TLG_LAYOUT_PLAIN(false, false)};

TLG_DEFINE_ERROR_WORD_READER(error_word_nn)

}  // namespace tlg
