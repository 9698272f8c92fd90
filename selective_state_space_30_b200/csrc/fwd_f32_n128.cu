// Instantiations of the forward-scan kernel for f32 I/O, N = 128 states.
#include "scan_kernel.cuh"

namespace ssm {
SSM_DEFINE_PICK(float, f32, 128)
}  // namespace ssm
