// Instantiations of the forward-scan kernel for bf16 I/O, N = 32 states.
#include "scan_kernel.cuh"

namespace ssm {
SSM_DEFINE_PICK(__nv_bfloat16, bf16, 32)
}  // namespace ssm
