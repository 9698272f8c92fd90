#pragma once
// The chunked tensor-core (SSD) forward for the per-head layout with dstate 128
// and head dim 64 (ssd.cu); plans dispatch to it where it applies.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ssm_scan.h"

namespace ssm {

struct SsdParams {
    const __nv_bfloat16* delta;   // (batch, nheads, seqlen)
    const float* A;               // (nheads)
    const float* D;               // (dim) or nullptr
    const float* bias;            // (nheads) or nullptr
    const __nv_bfloat16* z;       // (batch, dim, seqlen) or nullptr
    const float* h0;              // (batch, dim, dstate) or nullptr
    __nv_bfloat16* out;           // (batch, dim, seqlen)
    float* last_state;            // (batch, dim, dstate) or nullptr
    int* status;                  // kernel-side ssm_status_t
    int64_t batch, dim, seqlen, nheads, ngroups;
    int softplus;
    unsigned spin_limit;
};

// 2-D tensor maps (time x rows), 64-step boxes with the 128-byte swizzle:
// u, z and out rows (batch*dim) in boxes of 64 rows, B and C rows (batch*ngroups*dstate)
// in boxes of 128 rows; z is unused (and may be left zero) when there is no gate.
struct SsdMaps {
    CUtensorMap u, z, B, C, out;
};

// bf16 I/O, nheads < dim with dim/nheads == 64, dstate == 128, seqlen a positive multiple of 128.
bool ssd_eligible(const ssm_dims_t& d);
int ssd_smem_bytes();
// one CTA of 512 threads per (batch row, head): grid = batch * nheads
int ssd_launch(const SsdParams& prm, const SsdMaps& maps, int64_t grid, cudaStream_t s);

}  // namespace ssm
