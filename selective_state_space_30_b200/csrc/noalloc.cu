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
//  * Every call shares the one array.  Each call clears the part that must start
//    at zero (counters and flags) on its stream before its launch; calls whose
//    kernels overlap on the GPU (two streams at once) race on the array and
//    must not be made.
//  * Kernel-side conditions (a bounded wait that gave up) are recorded in the
//    array and cleared by the next call; this entry point does not report them.
//  * Nothing here calls cudaMalloc, cudaFree or any other allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
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

bool dims_valid(const ssm_dims_t* d) {
    if (!d) return false;
    if (d->batch < 0 || d->dim <= 0 || d->seqlen < 0 || d->dstate <= 0) return false;
    if (d->nheads <= 0 || d->ngroups <= 0) return false;
    if (d->dim % d->nheads || d->dim % d->ngroups) return false;
    if (d->io_dtype != SSM_F32 && d->io_dtype != SSM_BF16) return false;
    if (d->reserved != 0) return false;
    const int64_t lim = (int64_t)1 << 46;
    const int64_t L = d->seqlen > 0 ? d->seqlen : 1;
    if (d->batch > lim / d->dim || d->batch * d->dim > lim / L) return false;
    if (d->batch * d->ngroups > lim / (d->dstate * L)) return false;
    return true;
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encoder() {
    static std::atomic<EncodeFn> fn{nullptr};
    EncodeFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void* sym = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &sym, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeFn>(sym);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

bool encode(CUtensorMap* m, const void* base, int esz, uint64_t cols, uint64_t rows, uint32_t box_rows,
            CUtensorMapSwizzle swz) {
    EncodeFn enc = encoder();
    if (!enc || cols == 0 || rows == 0) return false;
    const cuuint64_t gdim[2] = {cols, rows};
    const cuuint64_t gstride[1] = {cols * (uint64_t)esz};
    const cuuint32_t box[2] = {(cuuint32_t)ssm::kTB, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int ssm_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                                              const void* C, const float* D, const void* z,
                                              const float* delta_bias, int softplus, const ssm_dims_t* dims,
                                              void* out, float* last_state, ssm_stream_t stream) {
    if (!dims_valid(dims)) return SSM_ERR_INVALID_ARG;
    const ssm_dims_t& d = *dims;
    if (d.batch > 0 && d.seqlen > 0 && (!u || !delta || !B || !C || !out)) return SSM_ERR_INVALID_ARG;
    if (!A) return SSM_ERR_INVALID_ARG;
    const bool head = d.nheads != d.dim;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
    void* scratch = nullptr;
    int sms = 0;
    const int rc = device_setup(dev, &scratch, &sms);
    if (rc != SSM_OK) return rc;
    if (d.batch == 0) return SSM_OK;

    // the schedule: the same policy as a plan (the default lane layout, one persistent CTA
    // per SM, the default segment length)
    const int64_t Dg = d.dim / d.ngroups;
    ssm::Layout lay;
    if (!ssm::choose_layout(d, sms, 0, 0, &lay)) return SSM_ERR_UNSUPPORTED;
    const int w = lay.w;
    const int ct = lay.v.ch_per_tile;
    const int64_t n_tiles = ssm::layout_tiles(d, ct);
    int64_t ctas = sms;
    const int64_t L = d.seqlen;
    const int64_t seg_len = ssm::default_seg_len(L, n_tiles, ctas);
    const int64_t n_seg = L > 0 ? (L + seg_len - 1) / seg_len : 1;
    const int64_t n_units = n_tiles * n_seg;
    if (n_units >= (int64_t)1 << 31) return SSM_ERR_UNSUPPORTED;
    if (ctas > n_units) ctas = n_units;

    // the workspace must fit the static scratch
    const size_t flags_off = 64;
    const size_t carry_off = (flags_off + (size_t)n_tiles * 4 + 255) / 256 * 256;
    const size_t need = carry_off + (size_t)n_tiles * ct * d.dstate * 4;
    if (need > kNoAllocScratchBytes) return SSM_ERR_UNSUPPORTED;

    // vector path (tensor maps) when rows are 16-byte aligned; else guarded element copies
    const int esz = d.io_dtype == SSM_BF16 ? 2 : 4;
    const int64_t P = d.dim / d.nheads;
    int delta_rows = ct;
    if (head) {
        delta_rows = (int)((ct - 1) / P + 2);
        if (delta_rows > ct) delta_rows = ct;
    }
    bool vec = L > 0 && L % 16 == 0 && a16(u) && a16(delta) && a16(B) && a16(C) && a16(out) && (!z || a16(z));
    ssm::TensorMaps tm;
    std::memset(&tm, 0, sizeof(tm));
    if (vec) {
        const CUtensorMapSwizzle bc = esz == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
        vec = encode(&tm.u, u, esz, L, d.batch * d.dim, ct, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode(&tm.delta, delta, esz, L, d.batch * d.nheads, delta_rows, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              (!z || encode(&tm.z, z, esz, L, d.batch * d.dim, ct, CU_TENSOR_MAP_SWIZZLE_NONE)) &&
              encode(&tm.B, B, esz, L, d.batch * d.ngroups * d.dstate, (uint32_t)d.dstate, bc) &&
              encode(&tm.C, C, esz, L, d.batch * d.ngroups * d.dstate, (uint32_t)d.dstate, bc);
    }
    ssm::Variant v;
    if (!ssm::pick_variant(d.io_dtype, d.dstate, head, vec, w, lay.spl, &v)) return SSM_ERR_UNSUPPORTED;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(scratch);
    // counters, status and flags start at zero on every call (the carry region needs no clearing)
    if (cudaMemsetAsync(ws, 0, carry_off, s) != cudaSuccess) return SSM_ERR_CUDA;
    ssm::FwdParams prm;
    prm.u = u; prm.delta = delta; prm.A = A; prm.B = B; prm.C = C; prm.D = D; prm.z = z;
    prm.bias = delta_bias; prm.h0 = nullptr; prm.out = out; prm.last_state = last_state;
    prm.ws = reinterpret_cast<ssm::WsHeader*>(ws);
    prm.flags = reinterpret_cast<unsigned*>(ws + flags_off);
    prm.carry = reinterpret_cast<float*>(ws + carry_off);
    prm.dim = d.dim; prm.seqlen = d.seqlen; prm.nheads = d.nheads; prm.ngroups = d.ngroups;
    prm.softplus = softplus ? 1 : 0;
    prm.tiles_per_group = (int)((Dg + ct - 1) / ct);
    prm.n_tiles = (int)n_tiles;
    prm.n_seg = (int)n_seg;
    prm.seg_len = (int)seg_len;
    prm.n_units = (unsigned)n_units;
    prm.n_ctas = (unsigned)ctas;
    prm.spin_limit = 1u << 21;
    prm.delta_rows = delta_rows;
    if (v.smem > 48 * 1024 &&
        cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    v.fn<<<(unsigned)ctas, v.threads, v.smem, s>>>(prm, tm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
