// Instantiations of the forward-scan kernel for f32 I/O, N = 16 states.
#include "scan_kernel.cuh"

namespace ssm {
SSM_DEFINE_PICK(float, f32, 16)
}  // namespace ssm
