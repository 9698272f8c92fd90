// Instantiations of the tensor-memory forward-scan kernel (bf16 I/O, N = 16 states).
#include "scan_kernel.cuh"

namespace ssm {
SSM_DEFINE_PICK_TC
}  // namespace ssm
