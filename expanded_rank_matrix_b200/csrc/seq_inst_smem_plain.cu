// Instantiates the sequential kernel for tiles held in shared memory, without the
// threshold variants and refinement sweeps (one unit per case, so the
// instantiations compile side by side).
#include "seq_kernel.cuh"

namespace externd {
EXTERND_SEQ_KERNELS(false, false, )
}  // namespace externd
