// One step of the selective-SSM recurrence with the state kept in HBM: the
// inference ("RNN-style", constant-size state) mode of the Mamba
// "architecture-details" page, sections "Parallel Algorithm" (sequential mode)
// and "Memory Efficiency" (inference).  Declared in include/ssm_scan.h as
// ssm_selective_state_update.
//
// The step is bound by HBM: every state row is read and written once, and the
// exps per element are a handful.  The state rows reach shared memory by bulk
// copies, so enough bytes are in flight to cover the HBM latency.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "scan_kernel.cuh"   // ex2_approx, softplus1, silu1, mbarrier and bulk-copy helpers
#include "ssm_scan.h"

namespace {

using ssm::ex2_approx;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 256;
constexpr int kMaxGridY = 65535;

template <typename T> __device__ __forceinline__ float ld_io(const T* p);
template <> __device__ __forceinline__ float ld_io<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st_io(T* p, float v);
template <> __device__ __forceinline__ void st_io<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void st_io<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

// four consecutive B or C values
template <typename T> __device__ __forceinline__ float4 ld4(const T* p);
template <> __device__ __forceinline__ float4 ld4<float>(const float* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
}
template <> __device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
    return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                       __uint_as_float(w.y & 0xFFFF0000u));
}

struct StepParams {
    float* state;
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *bias;
    void* out;
    int64_t batch;
    uint32_t dim, nheads, ngroups;
    uint32_t head_dim, group_dim;   // dim / nheads, dim / ngroups
    int softplus;
};

// grid.y walks the batch rows, grid.x the chunks of R = 4096/N channels of a
// row.  One thread bulk-copies the chunk's state rows (and, per channel, its A
// rows) into shared memory with cp.async.bulk: 16 KB of state in flight per CTA
// without holding registers, several CTAs per SM.  Then thread slots (channel,
// lane j) -- N/4 lanes per channel, four states per lane -- update the states in
// four passes and store them back with evict-first 16-byte stores; a warp covers
// contiguous 512-byte stretches.
template <int N>
struct StepCfg {
    static constexpr int TPC = N / 4;                 // lanes per channel
    static constexpr int R = 4096 / N;                // channels per CTA
    static constexpr int PASSES = R * TPC / kThreads; // slots per thread
    static constexpr int STATE_BYTES = R * N * 4;     // 16 KB
    static_assert(PASSES * kThreads == R * TPC, "whole passes");
};

template <typename T, int N>
__global__ void __launch_bounds__(kThreads, 6) state_update_kernel(const StepParams p) {
    using SC = StepCfg<N>;
    constexpr uint32_t TPC = SC::TPC;
    __shared__ __align__(128) float sh[SC::R * N];     // the chunk's states
    __shared__ __align__(128) float sa[SC::R * N];     // the chunk's A rows (per-channel layout)
    __shared__ __align__(8) uint64_t bar;
    const bool head = p.nheads != p.dim;
    const uint32_t d0 = blockIdx.x * (uint32_t)SC::R;
    const uint32_t nch = p.dim - d0 < (uint32_t)SC::R ? p.dim - d0 : (uint32_t)SC::R;
    const T* u = static_cast<const T*>(p.u);
    const T* dl = static_cast<const T*>(p.delta);
    if (threadIdx.x == 0) {
        ssm::mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    unsigned phase = 0;
    for (int64_t b = blockIdx.y; b < p.batch; b += gridDim.y, phase ^= 1u) {
        const int64_t c0 = b * p.dim + d0;
        if (threadIdx.x == 0) {
            const unsigned bytes = nch * N * 4u;
            ssm::mbar_arrive_tx(&bar, bytes * (head ? 1u : 2u));
            ssm::bulk_g2s(sh, p.state + c0 * N, bytes, &bar);
            if (!head) ssm::bulk_g2s(sa, p.A + (int64_t)d0 * N, bytes, &bar);
        }
        // per-slot inputs from global memory while the bulk copies are in flight (B and C
        // rows are shared by all channels of a group: they come from L1 in the passes below)
        float uu[SC::PASSES], x[SC::PASSES];
#pragma unroll
        for (int k = 0; k < SC::PASSES; ++k) {
            const uint32_t slot = threadIdx.x + (uint32_t)(k * kThreads);
            const uint32_t lc = slot / TPC;
            const uint32_t d = d0 + (lc < nch ? lc : 0u);
            const uint32_t hd = head ? d / p.head_dim : d;
            uu[k] = ld_io<T>(u + b * p.dim + d);
            x[k] = ld_io<T>(dl + b * p.nheads + hd) + (p.bias ? __ldg(p.bias + hd) : 0.f);
        }
        // the copies complete (they depend on nothing else; the wait is bounded all the same,
        // and a chunk that never arrived leaves its outputs NaN rather than hanging)
        bool ready = true;
        {
            const uint64_t t0 = ssm::now_ns();
            while (!ssm::mbar_try(&bar, phase)) {
                if (ssm::now_ns() - t0 > 1000000000ull) { ready = false; break; }
            }
        }
#pragma unroll
        for (int k = 0; k < SC::PASSES; ++k) {
            const uint32_t slot = threadIdx.x + (uint32_t)(k * kThreads);
            const uint32_t lc = slot / TPC;
            const bool live = lc < nch;
            const uint32_t d = d0 + (live ? lc : 0u);
            const uint32_t n0 = 4u * (slot % TPC);
            const int64_t c = b * p.dim + d;
            const uint32_t g = p.ngroups == 1 ? 0u : d / p.group_dim;
            const int64_t bc = (b * p.ngroups + g) * N + n0;
            const float4 bbk = ld4<T>(static_cast<const T*>(p.B) + bc);
            const float4 cck = ld4<T>(static_cast<const T*>(p.C) + bc);
            float4 a;
            if (head) {
                const float ah = __ldg(p.A + d / p.head_dim);
                a = make_float4(ah, ah, ah, ah);
            } else {
                a = *reinterpret_cast<const float4*>(sa + (live ? lc : 0u) * N + n0);
            }
            float4 hk = *reinterpret_cast<const float4*>(sh + (live ? lc : 0u) * N + n0);
            const float dt = p.softplus ? ssm::softplus1(x[k]) : x[k];
            const float du = dt * uu[k];
            const float s = dt * kLog2e;
            hk.x = fmaf(ex2_approx(s * a.x), hk.x, du * bbk.x);
            hk.y = fmaf(ex2_approx(s * a.y), hk.y, du * bbk.y);
            hk.z = fmaf(ex2_approx(s * a.z), hk.z, du * bbk.z);
            hk.w = fmaf(ex2_approx(s * a.w), hk.w, du * bbk.w);
            if (live && ready) __stcs(reinterpret_cast<float4*>(p.state + c * N + n0), hk);
            float y = fmaf(cck.x, hk.x, fmaf(cck.y, hk.y, fmaf(cck.z, hk.z, cck.w * hk.w)));
#pragma unroll
            for (uint32_t m = TPC / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
            if (live && n0 == 0) {
                y = fmaf(p.D ? __ldg(p.D + d) : 0.f, uu[k], y);
                if (p.z) y *= ssm::silu1(ld_io<T>(static_cast<const T*>(p.z) + c));
                st_io<T>(static_cast<T*>(p.out) + c, ready ? y : __int_as_float(0x7FC00000));
            }
        }
        // every thread is done with the chunk's shared copies before the next row's copies land
        __syncthreads();
    }
}

template <typename T>
int launch(const StepParams& prm, int64_t N, cudaStream_t s) {
    const int64_t R = 4096 / N;
    const int64_t bx = (prm.dim + R - 1) / R;
    const int64_t by = prm.batch < kMaxGridY ? prm.batch : kMaxGridY;
    if (bx == 0 || by == 0) return SSM_OK;
    const dim3 g((unsigned)bx, (unsigned)by);
    // shared memory holds the in-flight state: ask for the largest carveout
    static const bool carve = [] {
        cudaFuncSetAttribute(state_update_kernel<T, 8>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        cudaFuncSetAttribute(state_update_kernel<T, 16>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        cudaFuncSetAttribute(state_update_kernel<T, 32>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        cudaFuncSetAttribute(state_update_kernel<T, 64>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        cudaFuncSetAttribute(state_update_kernel<T, 128>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        return true;
    }();
    (void)carve;
    switch (N) {
        case 8: state_update_kernel<T, 8><<<g, kThreads, 0, s>>>(prm); break;
        case 16: state_update_kernel<T, 16><<<g, kThreads, 0, s>>>(prm); break;
        case 32: state_update_kernel<T, 32><<<g, kThreads, 0, s>>>(prm); break;
        case 64: state_update_kernel<T, 64><<<g, kThreads, 0, s>>>(prm); break;
        case 128: state_update_kernel<T, 128><<<g, kThreads, 0, s>>>(prm); break;
        default: return SSM_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int ssm_selective_state_update(const ssm_dims_t* dims, float* state, const void* u, const void* delta,
                                          const float* A, const void* B, const void* C, const float* D,
                                          const void* z, const float* delta_bias, int softplus, void* out,
                                          ssm_stream_t stream) {
    if (!dims) return SSM_ERR_INVALID_ARG;
    const ssm_dims_t& d = *dims;
    if (d.batch < 0 || d.dim <= 0 || d.dstate <= 0 || d.nheads <= 0 || d.ngroups <= 0 || d.reserved != 0)
        return SSM_ERR_INVALID_ARG;
    if (d.seqlen != 1 || d.dim % d.nheads || d.dim % d.ngroups) return SSM_ERR_INVALID_ARG;
    if (d.io_dtype != SSM_F32 && d.io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (d.batch > ((int64_t)1 << 40) / d.dim) return SSM_ERR_INVALID_ARG;
    const int64_t N = d.dstate;
    if (N != 8 && N != 16 && N != 32 && N != 64 && N != 128) return SSM_ERR_UNSUPPORTED;
    if (d.batch == 0) return SSM_OK;
    if (!state || !u || !delta || !A || !B || !C || !out) return SSM_ERR_INVALID_ARG;
    // four states per lane move as one 16-byte (state, A, fp32 B/C) or 8-byte (bf16 B/C) piece
    const uintptr_t bc_align = d.io_dtype == SSM_BF16 ? 8 : 16;
    if (!aligned(state, 16) || !aligned(B, bc_align) || !aligned(C, bc_align) ||
        (d.nheads == d.dim && !aligned(A, 16)))
        return SSM_ERR_UNSUPPORTED;
    // 32-bit index math within a batch row
    if (d.dim * (N / 4) >= ((int64_t)1 << 31)) return SSM_ERR_UNSUPPORTED;
    StepParams prm;
    prm.state = state; prm.u = u; prm.delta = delta; prm.B = B; prm.C = C; prm.z = z;
    prm.A = A; prm.D = D; prm.bias = delta_bias; prm.out = out;
    prm.batch = d.batch;
    prm.dim = (uint32_t)d.dim; prm.nheads = (uint32_t)d.nheads; prm.ngroups = (uint32_t)d.ngroups;
    prm.head_dim = (uint32_t)(d.dim / d.nheads); prm.group_dim = (uint32_t)(d.dim / d.ngroups);
    prm.softplus = softplus ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d.io_dtype == SSM_BF16 ? launch<__nv_bfloat16>(prm, N, s) : launch<float>(prm, N, s);
}
