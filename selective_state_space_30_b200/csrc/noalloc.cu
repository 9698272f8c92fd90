// ssm_selective_scan_fwd_noalloc: the forward scan for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a host
// framework that owns every byte of device memory through its own pre-reserved
// pool (a serving runtime with a fixed memory budget, a plugin host that forbids
// out-of-band allocations), or code that must not add an allocation, with its
// latency and its failure mode, to a hot path.  The plan-based entry points
// allocate their workspace in ssm_scan_plan; this one needs no plan and takes
// its scratch (scheduler counters, segment flags, segment carry states) from a
// fixed, statically sized __device__ array instead.
//
// Rules of use:
//  * The scratch array is kNoAllocScratchBytes (8 MiB) per device, held by every
//    GPU that loads the library until the process exits.  A problem whose
//    workspace does not fit is rejected with SSM_ERR_UNSUPPORTED before anything
//    is launched (roughly: batch * dim * dstate * 4 bytes of carry states must fit).
//  * The first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (once per device, with that device current); make that
//    first call before any stream capture.
//  * Under CUDA's lazy module loading (the default) the array, like the kernels,
//    is placed in device memory at that first call on each device, not when the
//    library is loaded.  A caller that reserves all of its device memory for its
//    own pool should make one warm-up call before reserving it, or run with
//    CUDA_MODULE_LOADING=EAGER.
//  * Every call shares the one array.  Each call clears the part that must start
//    at zero (counters, flags, status) on its stream before its launch; calls
//    whose kernels overlap on the GPU (two streams at once) race on the array
//    and must not be made.
//  * Kernel-side conditions (a bounded wait that gave up) are recorded in the
//    array's status word.  ssm_selective_scan_noalloc_device_status reads and
//    clears it; read it after a call and before the next one, which clears it.
//  * Nothing here calls cudaMalloc, cudaFree or any other allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cstring>

#include "layout.h"
#include "scan_kernel.cuh"
#include "ssm_scan.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

// The scratch: [0, 64) header | flags[n_tiles] | carry[n_tiles][CT][N] fp32.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host-side cache of the array's device address and the SM count, per device.
// (In host code the array's name is only a host-side stand-in, never a device address.)
std::atomic<int> g_ready[kMaxDevices];
void* g_scratch_addr[kMaxDevices];
int g_sm_count[kMaxDevices];

int device_setup(int dev, void** addr, int* sms) {
    if (dev < 0 || dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;
    if (g_ready[dev].load(std::memory_order_acquire) != 2) {
        int expected = 0;
        if (g_ready[dev].compare_exchange_strong(expected, 1, std::memory_order_acq_rel)) {
            void* p = nullptr;
            int n = 0;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess ||
                cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                g_ready[dev].store(0, std::memory_order_release);
                return SSM_ERR_CUDA;
            }
            g_scratch_addr[dev] = p;
            g_sm_count[dev] = n;
            g_ready[dev].store(2, std::memory_order_release);
        } else {
            while (g_ready[dev].load(std::memory_order_acquire) == 1) {
            }
            if (g_ready[dev].load(std::memory_order_acquire) != 2) return SSM_ERR_CUDA;
        }
    }
    *addr = g_scratch_addr[dev];
    *sms = g_sm_count[dev];
    return SSM_OK;
}

// Test hooks: make the chained waits of the next calls wait for a flag nobody sets,
// and bound every wait by a spin limit (0 = the default).
std::atomic<unsigned> g_hook_stall{0};
std::atomic<unsigned> g_hook_spin{0};
constexpr unsigned kDefaultSpin = 1u << 21;  // ~0.5 s of polling before a wait gives up

}  // namespace

extern "C" int ssm_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                                              const void* C, const float* D, const void* z,
                                              const float* delta_bias, int softplus, const ssm_dims_t* dims,
                                              void* out, float* last_state, ssm_stream_t stream) {
    if (!ssm::dims_ok(dims)) return SSM_ERR_INVALID_ARG;
    const ssm_dims_t& d = *dims;
    if (d.batch > 0 && d.seqlen > 0 && (!u || !delta || !B || !C || !out)) return SSM_ERR_INVALID_ARG;
    if (!A) return SSM_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    void* scratch = nullptr;
    int sms = 0;
    int rc = device_setup(dev, &scratch, &sms);
    if (rc != SSM_OK) return rc;
    if (d.batch == 0) return SSM_OK;

    // the schedule of a plan with default options (the same code as the plan path)
    ssm::FwdGeom g;
    rc = ssm::fwd_geometry(d, sms, 0, 0, 0, 0, 0, 0, &g);
    if (rc != SSM_OK) return rc;
    // the workspace must fit the static scratch
    if (g.ws_bytes > kNoAllocScratchBytes) return SSM_ERR_UNSUPPORTED;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(scratch);
    // counters, status and flags start at zero on every call (the carry region needs no clearing)
    if (cudaMemsetAsync(ws, 0, g.carry_off, s) != cudaSuccess) return SSM_ERR_CUDA;
    if (g_hook_stall.load() &&
        cudaMemsetAsync(ws + offsetof(ssm::WsHeader, inject), 1, 1, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    const unsigned spin = g_hook_spin.load() ? g_hook_spin.load() : kDefaultSpin;
    const ssm::FwdArgs a{u, delta, A, B, C, D, z, delta_bias, softplus, nullptr, out, last_state};
    return ssm::fwd_launch(d, g, a, ws, spin, s);
}

extern "C" int ssm_selective_scan_noalloc_device_status(ssm_stream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    void* scratch = nullptr;
    int sms = 0;
    const int rc = device_setup(dev, &scratch, &sms);
    if (rc != SSM_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* status = reinterpret_cast<int*>(static_cast<unsigned char*>(scratch) + offsetof(ssm::WsHeader, status));
    int st = SSM_OK;
    if (cudaMemcpyAsync(&st, status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (st != SSM_OK && (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess ||
                         cudaStreamSynchronize(s) != cudaSuccess))
        return SSM_ERR_CUDA;
    return st;
}

extern "C" int ssm_selective_scan_noalloc_test_hooks(int stall, int64_t spin_limit) {
    if (spin_limit < 0 || spin_limit > 0x7fffffff) return SSM_ERR_INVALID_ARG;
    g_hook_stall.store(stall ? 1u : 0u);
    g_hook_spin.store((unsigned)spin_limit);
    return SSM_OK;
}
