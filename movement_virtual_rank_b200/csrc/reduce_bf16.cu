// Reduction kernels instantiated for one element type (see reduce_impl.cuh).
#include "reduce_impl.cuh"

MVR_REDUCE_INSTANCE(bf16, COLL_BF16)
