// Block-ALS path (filled in by the block kernels).
#include "../../include/externd.h"
#include "internal.h"

namespace externd {

int block_decompose(const BlockHostArgs&, cudaStream_t) { return EXTERND_ERR_INVALID_ARG; }

}  // namespace externd
