// C ABI of the selective-scan library (declared in include/ssm_scan.h):
// argument checks, plans, kernel choice and launch.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>

#include "scan_kernel.cuh"
#include "ssm_scan.h"

namespace ssm {

// MUFU ex2 throughput probe: 16 independent dependency chains per thread.
__global__ void __launch_bounds__(256) probe_ex2_kernel(float* sink, int iters) {
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = -0.001f * (threadIdx.x + i);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = ex2_approx(x[i]) - 1.0f;
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) s += x[i];
    sink[blockIdx.x * 256 + threadIdx.x] = s;
}

static bool pick_variant(int dtype, int64_t N, bool head, bool vec, Variant* v) {
    const bool bf = dtype == SSM_BF16;
    switch (N) {
        case 8: return bf ? pick_bf16_n8(head, vec, v) : pick_f32_n8(head, vec, v);
        case 16: return bf ? pick_bf16_n16(head, vec, v) : pick_f32_n16(head, vec, v);
        case 32: return bf ? pick_bf16_n32(head, vec, v) : pick_f32_n32(head, vec, v);
        case 64: return bf ? pick_bf16_n64(head, vec, v) : pick_f32_n64(head, vec, v);
        case 128: return bf ? pick_bf16_n128(head, vec, v) : pick_f32_n128(head, vec, v);
        default: return false;
    }
}

}  // namespace ssm

// ------------------------------------------------------------------- C ABI

struct ssm_plan_s {
    uint32_t magic;
    ssm_dims_t dims;
    int device;
    int* d_status;
    // lazily allocated device mirrors for the host-buffer entry point
    void* h_bufs[11];
    size_t h_sizes[11];
};

namespace {
constexpr uint32_t kMagic = 0x53534d31u;  // "SSM1"
constexpr uint32_t kDead = 0xdeadbeefu;

bool dims_ok(const ssm_dims_t* d) {
    if (!d) return false;
    if (d->batch < 0 || d->dim <= 0 || d->seqlen < 0 || d->dstate <= 0) return false;
    if (d->nheads <= 0 || d->ngroups <= 0) return false;
    if (d->dim % d->nheads || d->dim % d->ngroups) return false;
    if (d->io_dtype != SSM_F32 && d->io_dtype != SSM_BF16) return false;
    if (d->reserved != 0) return false;
    // element offsets must fit the kernel's 64-bit arithmetic comfortably
    const int64_t lim = (int64_t)1 << 46;
    if (d->batch > lim / d->dim || d->batch * d->dim > lim / (d->seqlen > 0 ? d->seqlen : 1)) return false;
    if (d->batch * d->ngroups > lim / (d->dstate * (d->seqlen > 0 ? d->seqlen : 1))) return false;
    return true;
}

bool same_dims(const ssm_dims_t* a, const ssm_dims_t* b) {
    return a->batch == b->batch && a->dim == b->dim && a->seqlen == b->seqlen && a->dstate == b->dstate &&
           a->nheads == b->nheads && a->ngroups == b->ngroups && a->io_dtype == b->io_dtype;
}

bool plan_ok(const ssm_plan_t p) { return p && p->magic == kMagic; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int tiles_per_group(const ssm_dims_t& d, int ch) {
    const int64_t Dg = d.dim / d.ngroups;
    return (int)((Dg + ch - 1) / ch);
}

int64_t grid_of(const ssm_dims_t& d, int ch) { return d.batch * d.ngroups * tiles_per_group(d, ch); }

int set_device(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return SSM_ERR_CUDA;
    if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return SSM_ERR_CUDA;
    return SSM_OK;
}

int launch_fwd(ssm_plan_t plan, const void* u, const void* delta, const float* A, const void* B, const void* C,
               const float* D, const void* z, const float* delta_bias, int softplus, const float* h0, void* out,
               float* last_state, cudaStream_t stream) {
    const ssm_dims_t& d = plan->dims;
    const bool head = d.nheads != d.dim;
    // Vector loads/stores need every per-lane chunk (up to 16 elements) wholly
    // inside or outside a row and 16-byte aligned: L % 16 == 0 plus aligned bases.
    const bool vec = (d.seqlen % 16 == 0) && aligned16(u) && aligned16(delta) && aligned16(B) &&
                     aligned16(C) && aligned16(out) && (!z || aligned16(z));
    ssm::Variant v;
    if (!ssm::pick_variant(d.io_dtype, d.dstate, head, vec, &v)) return SSM_ERR_UNSUPPORTED;
    if (d.batch == 0) return SSM_OK;
    ssm::FwdParams prm;
    prm.u = u; prm.delta = delta; prm.A = A; prm.B = B; prm.C = C; prm.D = D; prm.z = z;
    prm.bias = delta_bias; prm.h0 = h0; prm.out = out; prm.last_state = last_state; prm.status = plan->d_status;
    prm.batch = d.batch; prm.dim = d.dim; prm.seqlen = d.seqlen; prm.nheads = d.nheads; prm.ngroups = d.ngroups;
    prm.softplus = softplus ? 1 : 0;
    prm.tiles_per_group = tiles_per_group(d, v.ch_per_cta);
    const int64_t grid = grid_of(d, v.ch_per_cta);
    if (grid > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
    if (v.smem > 48 * 1024) {
        if (cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem) != cudaSuccess)
            return SSM_ERR_CUDA;
    }
    v.fn<<<(unsigned)grid, ssm::kThreads, v.smem, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
}  // namespace

extern "C" {

const char* ssm_status_string(int status) {
    switch (status) {
        case SSM_OK: return "ok";
        case SSM_ERR_INVALID_ARG: return "invalid argument";
        case SSM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case SSM_ERR_CUDA: return "CUDA runtime error";
        case SSM_ERR_TIMEOUT: return "device-side bounded wait timed out";
        case SSM_ERR_BOUNDS: return "device-side bounds check failed";
        default: return "unknown status";
    }
}

int ssm_scan_plan(ssm_plan_t* out_plan, const ssm_dims_t* dims, int device) {
    if (!out_plan) return SSM_ERR_INVALID_ARG;
    *out_plan = nullptr;
    if (!dims_ok(dims)) return SSM_ERR_INVALID_ARG;
    ssm::Variant v;
    if (!ssm::pick_variant(dims->io_dtype, dims->dstate, dims->nheads != dims->dim, true, &v))
        return SSM_ERR_UNSUPPORTED;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return SSM_ERR_CUDA;
    if (set_device(device) != SSM_OK) return SSM_ERR_CUDA;
    ssm_plan_s* p = new (std::nothrow) ssm_plan_s();
    if (!p) return SSM_ERR_CUDA;
    p->magic = kMagic;
    p->dims = *dims;
    p->device = device;
    if (cudaMalloc(&p->d_status, sizeof(int)) != cudaSuccess) {
        delete p;
        return SSM_ERR_CUDA;
    }
    if (cudaMemset(p->d_status, 0, sizeof(int)) != cudaSuccess) {
        cudaFree(p->d_status);
        delete p;
        return SSM_ERR_CUDA;
    }
    *out_plan = p;
    return SSM_OK;
}

int ssm_selective_scan_fwd_h0(ssm_plan_t plan, const void* u, const void* delta, const float* A, const void* B,
                              const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                              const ssm_dims_t* dims, const float* h0, void* out, float* last_state,
                              ssm_stream_t stream) {
    if (!plan_ok(plan) || !dims || !same_dims(dims, &plan->dims)) return SSM_ERR_INVALID_ARG;
    if (plan->dims.batch > 0 && plan->dims.seqlen > 0 && (!u || !delta || !B || !C || !out)) return SSM_ERR_INVALID_ARG;
    if (!A) return SSM_ERR_INVALID_ARG;
    if (set_device(plan->device) != SSM_OK) return SSM_ERR_CUDA;
    return launch_fwd(plan, u, delta, A, B, C, D, z, delta_bias, softplus, h0, out, last_state,
                      reinterpret_cast<cudaStream_t>(stream));
}

int ssm_selective_scan_fwd(ssm_plan_t plan, const void* u, const void* delta, const float* A, const void* B,
                           const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                           const ssm_dims_t* dims, void* out, float* last_state, ssm_stream_t stream) {
    return ssm_selective_scan_fwd_h0(plan, u, delta, A, B, C, D, z, delta_bias, softplus, dims, nullptr, out,
                                     last_state, stream);
}

int ssm_selective_scan_fwd_host(ssm_plan_t plan, const void* u, const void* delta, const float* A, const void* B,
                                const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                                const ssm_dims_t* dims, void* out, float* last_state, ssm_stream_t stream) {
    if (!plan_ok(plan) || !dims || !same_dims(dims, &plan->dims)) return SSM_ERR_INVALID_ARG;
    const ssm_dims_t& d = plan->dims;
    if (!u || !delta || !A || !B || !C || !out) return SSM_ERR_INVALID_ARG;
    if (set_device(plan->device) != SSM_OK) return SSM_ERR_CUDA;
    const size_t e = d.io_dtype == SSM_BF16 ? 2 : 4;
    const size_t n_bdl = (size_t)(d.batch * d.dim * d.seqlen);
    const size_t n_bhl = (size_t)(d.batch * d.nheads * d.seqlen);
    const size_t n_bc = (size_t)(d.batch * d.ngroups * d.dstate * d.seqlen);
    const size_t n_a = (size_t)(d.nheads == d.dim ? d.dim * d.dstate : d.nheads);
    const size_t n_state = (size_t)(d.batch * d.dim * d.dstate);
    // slots: 0 u, 1 delta, 2 A, 3 B, 4 C, 5 D, 6 z, 7 bias, 8 out, 9 last_state
    const void* src[10] = {u, delta, A, B, C, D, z, delta_bias, nullptr, nullptr};
    const size_t bytes[10] = {n_bdl * e, n_bhl * e, n_a * 4, n_bc * e, n_bc * e, (size_t)d.dim * 4, n_bdl * e,
                              (size_t)d.nheads * 4, n_bdl * e, n_state * 4};
    const bool used[10] = {true, true, true, true, true, D != nullptr, z != nullptr, delta_bias != nullptr, true,
                           last_state != nullptr};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < 10; ++i) {
        if (!used[i]) continue;
        if (plan->h_sizes[i] < bytes[i]) {
            if (plan->h_bufs[i]) cudaFree(plan->h_bufs[i]);
            plan->h_bufs[i] = nullptr;
            plan->h_sizes[i] = 0;
            if (bytes[i] && cudaMalloc(&plan->h_bufs[i], bytes[i]) != cudaSuccess) return SSM_ERR_CUDA;
            plan->h_sizes[i] = bytes[i];
        }
        if (i < 8 && bytes[i] &&
            cudaMemcpyAsync(plan->h_bufs[i], src[i], bytes[i], cudaMemcpyHostToDevice, s) != cudaSuccess)
            return SSM_ERR_CUDA;
    }
    int rc = launch_fwd(plan, plan->h_bufs[0], plan->h_bufs[1], (const float*)plan->h_bufs[2], plan->h_bufs[3],
                        plan->h_bufs[4], D ? (const float*)plan->h_bufs[5] : nullptr, z ? plan->h_bufs[6] : nullptr,
                        delta_bias ? (const float*)plan->h_bufs[7] : nullptr, softplus, nullptr, plan->h_bufs[8],
                        last_state ? (float*)plan->h_bufs[9] : nullptr, s);
    if (rc != SSM_OK) return rc;
    if (bytes[8] && cudaMemcpyAsync(out, plan->h_bufs[8], bytes[8], cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (last_state && bytes[9] &&
        cudaMemcpyAsync(last_state, plan->h_bufs[9], bytes[9], cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    return SSM_OK;
}

int ssm_scan_destroy(ssm_plan_t plan) {
    if (!plan) return SSM_OK;
    if (!plan_ok(plan)) return SSM_ERR_INVALID_ARG;
    set_device(plan->device);
    cudaDeviceSynchronize();
    cudaFree(plan->d_status);
    for (int i = 0; i < 11; ++i)
        if (plan->h_bufs[i]) cudaFree(plan->h_bufs[i]);
    plan->magic = kDead;
    delete plan;
    return SSM_OK;
}

int ssm_scan_device_status(ssm_plan_t plan, ssm_stream_t stream) {
    if (!plan_ok(plan)) return SSM_ERR_INVALID_ARG;
    if (set_device(plan->device) != SSM_OK) return SSM_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int h = 0;
    if (cudaMemcpyAsync(&h, plan->d_status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SSM_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSM_ERR_CUDA;
    if (cudaMemsetAsync(plan->d_status, 0, sizeof(int), s) != cudaSuccess) return SSM_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSM_ERR_CUDA;
    return h;
}

int ssm_scan_plan_info(ssm_plan_t plan, int* grid, int* block, int* smem_bytes, int* launches_per_call,
                       const char** variant) {
    if (!plan_ok(plan)) return SSM_ERR_INVALID_ARG;
    const ssm_dims_t& d = plan->dims;
    ssm::Variant v;
    if (!ssm::pick_variant(d.io_dtype, d.dstate, d.nheads != d.dim, d.seqlen % 16 == 0, &v))
        return SSM_ERR_UNSUPPORTED;
    if (grid) *grid = (int)grid_of(d, v.ch_per_cta);
    if (block) *block = ssm::kThreads;
    if (smem_bytes) *smem_bytes = v.smem;
    if (launches_per_call) *launches_per_call = d.batch > 0 ? 1 : 0;
    if (variant) *variant = v.name;
    return SSM_OK;
}

int ssm_probe_ex2(float* sink, int blocks, int iters, ssm_stream_t stream) {
    if (!sink || blocks <= 0 || iters <= 0) return SSM_ERR_INVALID_ARG;
    ssm::probe_ex2_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(sink, iters);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
