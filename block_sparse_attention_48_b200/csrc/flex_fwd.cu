// Base instances of the block-sparse FlexAttention forward kernel (no work-order
// ranking, no paged K / V in their code) and the launch dispatch; the kernel body
// is in flex_fwd_impl.cuh.
#define FWD_EXT 0
#include "flex_fwd_impl.cuh"
