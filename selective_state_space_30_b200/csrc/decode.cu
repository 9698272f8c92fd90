// One step of the selective-SSM recurrence with the state kept in HBM: the
// inference ("RNN-style", constant-size state) mode of the Mamba
// "architecture-details" page, sections "Parallel Algorithm" (sequential mode)
// and "Memory Efficiency" (inference).  Declared in include/ssm_scan.h as
// ssm_selective_state_update.
//
// The step is bound by HBM: every state row is read and written once, and the
// exps per element are a handful.  Layout: TPC = N/4 lanes per channel, four
// consecutive states per lane, so a warp reads and writes its state rows as
// contiguous 16-byte pieces; the lanes of a channel sum y with shuffles.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ssm_scan.h"

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 256;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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
    int64_t batch, dim, nheads, ngroups;
    int softplus;
};

template <typename T, int N>
__global__ void __launch_bounds__(kThreads) state_update_kernel(const StepParams p) {
    constexpr int TPC = N / 4;   // lanes per channel
    const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t ch = gid / TPC;           // flat (b, d)
    const int j = (int)(gid % TPC);
    const bool live = ch < p.batch * p.dim;
    const int64_t c = live ? ch : 0;
    const int64_t b = c / p.dim, d = c % p.dim;
    const int64_t hd = d / (p.dim / p.nheads), g = d / (p.dim / p.ngroups);
    const bool head = p.nheads != p.dim;
    const T* u = static_cast<const T*>(p.u);
    const T* dl = static_cast<const T*>(p.delta);
    const float uu = ld_io<T>(u + c);
    float x = ld_io<T>(dl + b * p.nheads + hd) + (p.bias ? __ldg(p.bias + hd) : 0.f);
    // softplus(x) = max(x, 0) + log1p(exp(-|x|))
    const float dt = p.softplus ? fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x))) : x;
    const float du = dt * uu;
    const int n0 = 4 * j;
    const float4 bb = ld4<T>(static_cast<const T*>(p.B) + (b * p.ngroups + g) * N + n0);
    const float4 cc = ld4<T>(static_cast<const T*>(p.C) + (b * p.ngroups + g) * N + n0);
    float4 a;
    if (head) {
        const float ah = __ldg(p.A + hd);
        a = make_float4(ah, ah, ah, ah);
    } else {
        a = __ldg(reinterpret_cast<const float4*>(p.A + d * N + n0));
    }
    float4* hp = reinterpret_cast<float4*>(p.state + c * N + n0);
    float4 h = live ? *hp : make_float4(0.f, 0.f, 0.f, 0.f);
    h.x = fmaf(ex2_approx(dt * a.x * kLog2e), h.x, du * bb.x);
    h.y = fmaf(ex2_approx(dt * a.y * kLog2e), h.y, du * bb.y);
    h.z = fmaf(ex2_approx(dt * a.z * kLog2e), h.z, du * bb.z);
    h.w = fmaf(ex2_approx(dt * a.w * kLog2e), h.w, du * bb.w);
    if (live) *hp = h;
    float y = fmaf(cc.x, h.x, fmaf(cc.y, h.y, fmaf(cc.z, h.z, cc.w * h.w)));
#pragma unroll
    for (int m = TPC / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
    if (live && j == 0) {
        y = fmaf(p.D ? __ldg(p.D + d) : 0.f, uu, y);
        if (p.z) {
            const float zz = ld_io<T>(static_cast<const T*>(p.z) + c);
            y *= zz / (1.f + __expf(-zz));
        }
        st_io<T>(static_cast<T*>(p.out) + c, y);
    }
}

template <typename T>
int launch(const StepParams& prm, int64_t N, cudaStream_t s) {
    const int64_t threads = prm.batch * prm.dim * (N / 4);
    const int64_t blocks = (threads + kThreads - 1) / kThreads;
    if (blocks > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    if (blocks == 0) return SSM_OK;
    switch (N) {
        case 8: state_update_kernel<T, 8><<<(unsigned)blocks, kThreads, 0, s>>>(prm); break;
        case 16: state_update_kernel<T, 16><<<(unsigned)blocks, kThreads, 0, s>>>(prm); break;
        case 32: state_update_kernel<T, 32><<<(unsigned)blocks, kThreads, 0, s>>>(prm); break;
        case 64: state_update_kernel<T, 64><<<(unsigned)blocks, kThreads, 0, s>>>(prm); break;
        case 128: state_update_kernel<T, 128><<<(unsigned)blocks, kThreads, 0, s>>>(prm); break;
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
    StepParams prm;
    prm.state = state; prm.u = u; prm.delta = delta; prm.B = B; prm.C = C; prm.z = z;
    prm.A = A; prm.D = D; prm.bias = delta_bias; prm.out = out;
    prm.batch = d.batch; prm.dim = d.dim; prm.nheads = d.nheads; prm.ngroups = d.ngroups;
    prm.softplus = softplus ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d.io_dtype == SSM_BF16 ? launch<__nv_bfloat16>(prm, N, s) : launch<float>(prm, N, s);
}
