// Causal depthwise convolution over time in front of the scan: the local
// convolution of the Mamba "architecture-details" page ("Model Configuration":
// d_conv, conv_bias; "Parameter Impact": the local context window before the
// SSM).  Declared in include/ssm_scan.h as ssm_causal_conv1d_fwd.
//
//   out[b,d,t] = act(bias[d] + sum_{k<width} w[d,k] * x[b,d,t-width+1+k]),  x = 0 before t = 0
//
// HBM-bound: each element is read and written once.  The row is cut into
// 16-byte chunks (8 bf16 or 4 fp32 steps); a lane computes four chunks, 32
// chunks apart, reading for each also the chunk before it for the width-1
// earlier steps.
// Rows whose length or base is not 16-byte aligned take a one-step-per-thread
// path with the same arithmetic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "scan_kernel.cuh"   // silu1
#include "ssm_scan.h"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxWidth = 4;

struct ConvParams {
    const void* x;
    const float* w;
    const float* bias;
    void* out;
    int64_t rows, seqlen, dim;
    int width;
    int silu;
};

template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int V = 4;   // steps per 16-byte chunk
    __device__ static void unpack(const uint4& q, float (&v)[V]) {
        v[0] = __uint_as_float(q.x); v[1] = __uint_as_float(q.y);
        v[2] = __uint_as_float(q.z); v[3] = __uint_as_float(q.w);
    }
    __device__ static uint4 pack(const float (&v)[V]) {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
    }
    __device__ static float load1(const void* p, int64_t i) { return __ldg(static_cast<const float*>(p) + i); }
    __device__ static void store1(void* p, int64_t i, float v) { static_cast<float*>(p)[i] = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int V = 8;
    __device__ static void unpack(const uint4& q, float (&v)[V]) {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ static uint4 pack(const float (&v)[V]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&b);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ static float load1(const void* p, int64_t i) {
        return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    }
    __device__ static void store1(void* p, int64_t i, float v) {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    }
};

template <int W>
__device__ __forceinline__ void taps(const ConvParams& p, int64_t d, float (&w)[W], float& b) {
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = __ldg(p.w + d * W + k);
    b = p.bias ? __ldg(p.bias + d) : 0.f;
}

// 16-byte chunks: chunk c of row r covers steps [c*V, c*V + V).  A warp owns a
// tile of 32*CPC consecutive chunks of a row; lane l takes chunks l, l+32, ...,
// so every load and store instruction of the warp covers 512 contiguous bytes.
// Each chunk also needs the chunk before it for the earlier taps (mostly an L1
// hit: it is the neighbour lane's chunk).  All loads are issued first.  W (the
// width) is a template parameter so every tap index is known at compile time.
constexpr int kCPC = 4;   // chunks per lane

template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv1d_vec_kernel(const ConvParams p) {
    using E = Elem<T>;
    constexpr int V = E::V;
    static_assert(W - 1 <= V, "the earlier steps fit in the previous chunk");
    const int64_t chunks = p.seqlen / V;
    const int64_t tiles = (chunks + 32 * kCPC - 1) / (32 * kCPC);   // warp tiles per row
    const int64_t wid = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= p.rows * tiles) return;
    const int64_t r = wid / tiles, c0 = (wid % tiles) * (32 * kCPC) + lane;
    float w[W], b;
    taps<W>(p, r % p.dim, w, b);
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const char*>(p.x) + r * p.seqlen * sizeof(T));
    uint4* orow = reinterpret_cast<uint4*>(static_cast<char*>(p.out) + r * p.seqlen * sizeof(T));
    uint4 cur_raw[kCPC], prev_raw[kCPC];
#pragma unroll
    for (int q = 0; q < kCPC; ++q) {
        const int64_t c = c0 + 32 * q;
        const bool in = c < chunks;
        cur_raw[q] = in ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        prev_raw[q] = in && c > 0 ? __ldg(xr + c - 1) : make_uint4(0u, 0u, 0u, 0u);   // zero bits are 0.0
    }
#pragma unroll
    for (int q = 0; q < kCPC; ++q) {
        const int64_t c = c0 + 32 * q;
        // steps of the previous chunk, then this one
        float xv[2 * V];
        {
            float prev[V], cur[V];
            E::unpack(prev_raw[q], prev);
            E::unpack(cur_raw[q], cur);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                xv[i] = prev[i];
                xv[V + i] = cur[i];
            }
        }
        float o[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            float v = b;
#pragma unroll
            for (int k = 0; k < W; ++k) v = fmaf(w[k], xv[V + i - (W - 1) + k], v);
            o[i] = p.silu ? ssm::silu1(v) : v;
        }
        if (c < chunks) orow[c] = E::pack(o);
    }
}

// one step per thread
template <typename T, int W>
__global__ void __launch_bounds__(kThreads) conv1d_scalar_kernel(const ConvParams p) {
    using E = Elem<T>;
    const int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (g >= p.rows * p.seqlen) return;
    const int64_t r = g / p.seqlen, t = g % p.seqlen;
    float w[W], b;
    taps<W>(p, r % p.dim, w, b);
    float v = b;
#pragma unroll
    for (int k = 0; k < W; ++k) {
        const int64_t s = t - (W - 1) + k;
        if (s >= 0) v = fmaf(w[k], E::load1(p.x, r * p.seqlen + s), v);
    }
    E::store1(p.out, g, p.silu ? ssm::silu1(v) : v);
}

template <typename T, int W>
int launch_w(const ConvParams& p, bool vec, cudaStream_t s) {
    // vector path: one warp per tile of 32*kCPC chunks
    const int64_t work = vec ? p.rows * ((p.seqlen / Elem<T>::V + 32 * kCPC - 1) / (32 * kCPC)) * 32
                             : p.rows * p.seqlen;
    const int64_t blocks = (work + kThreads - 1) / kThreads;
    if (blocks == 0) return SSM_OK;
    if (blocks > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    if (vec) conv1d_vec_kernel<T, W><<<(unsigned)blocks, kThreads, 0, s>>>(p);
    else conv1d_scalar_kernel<T, W><<<(unsigned)blocks, kThreads, 0, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <typename T>
int launch(const ConvParams& p, bool vec, cudaStream_t s) {
    switch (p.width) {
        case 1: return launch_w<T, 1>(p, vec, s);
        case 2: return launch_w<T, 2>(p, vec, s);
        case 3: return launch_w<T, 3>(p, vec, s);
        case 4: return launch_w<T, 4>(p, vec, s);
        default: return SSM_ERR_UNSUPPORTED;
    }
}

}  // namespace

extern "C" int ssm_causal_conv1d_fwd(int64_t batch, int64_t dim, int64_t seqlen, int32_t width, int32_t io_dtype,
                                     const void* x, const float* w, const float* bias, int silu, void* out,
                                     ssm_stream_t stream) {
    if (batch < 0 || dim <= 0 || seqlen < 0) return SSM_ERR_INVALID_ARG;
    if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (width < 1 || width > kMaxWidth) return SSM_ERR_UNSUPPORTED;
    if (batch > ((int64_t)1 << 46) / dim || (seqlen > 0 && batch * dim > ((int64_t)1 << 46) / seqlen))
        return SSM_ERR_INVALID_ARG;
    if (batch == 0 || seqlen == 0) return SSM_OK;
    if (!x || !w || !out) return SSM_ERR_INVALID_ARG;
    ConvParams p;
    p.x = x; p.w = w; p.bias = bias; p.out = out;
    p.rows = batch * dim; p.seqlen = seqlen; p.dim = dim; p.width = width; p.silu = silu ? 1 : 0;
    const int esz = io_dtype == SSM_BF16 ? 2 : 4;
    const int V = 16 / esz;
    const bool vec = seqlen % V == 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return io_dtype == SSM_BF16 ? launch<__nv_bfloat16>(p, vec, s) : launch<float>(p, vec, s);
}
