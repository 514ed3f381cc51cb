// Extended instances of the block-sparse FlexAttention forward kernel: the
// longest-first ranking of BlockMask rows and paged K / V compiled in (masks with
// a DOCUMENT leaf, fa_forward_paged); the kernel body is in flex_fwd_impl.cuh.
#define FWD_EXT 3  // kExtRank | kExtPage
#include "flex_fwd_impl.cuh"
