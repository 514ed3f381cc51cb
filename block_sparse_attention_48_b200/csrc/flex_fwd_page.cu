// Paged instances of the block-sparse FlexAttention forward kernel: the
// page-table read of paged K / V compiled in, the base work order (fa_forward_paged
// without a DOCUMENT leaf); the kernel body is in flex_fwd_impl.cuh.
#define FWD_EXT 2  // kExtPage
#include "flex_fwd_impl.cuh"
