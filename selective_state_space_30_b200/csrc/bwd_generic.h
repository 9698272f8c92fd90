// The backward scan for the shapes the tiled backward kernel does not cover: the
// per-head layout (one scalar A per head, delta and delta_bias per head) and every
// dstate in {8, 16, 32, 64, 128}.  Declared for bwd.cu, which dispatches to it.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "ssm_scan.h"

namespace ssm {

// SSM_OK when the generic backward covers `d` (dims already checked for consistency).
int bwd_generic_supported(const ssm_dims_t& d);

// Bytes of caller workspace the generic backward needs for `d`.
int64_t bwd_generic_workspace_bytes(const ssm_dims_t& d);

// Launch it on `s`: the workspace's first 8 bytes are the ticket / status header that
// ssm_selective_scan_bwd_device_status reads (always SSM_OK here: the kernel has no
// waits).  Arguments as ssm_selective_scan_bwd.
int bwd_generic_launch(const ssm_dims_t& d, const void* u, const void* delta, const float* A, const void* B,
                       const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                       const float* h0, const void* dout, const float* dlast, const ssm_grads_t& g,
                       unsigned char* ws, cudaStream_t s);

}  // namespace ssm
