// Instantiations of the forward-scan kernel for f32 I/O, N = 64 states.
#include "scan_kernel.cuh"

namespace ssm {
SSM_DEFINE_PICK(float, f32, 64)
}  // namespace ssm
