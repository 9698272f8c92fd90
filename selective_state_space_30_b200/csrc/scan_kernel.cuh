#pragma once
// Selective-SSM (S6) forward scan kernel for B200 (sm_100a): the template.
//
// What it computes is stated in include/ssm_scan.h (the recurrence of the
// Mamba "architecture-details" page, section "How S6 Works", with
// A_bar = exp(dt*A) from the "Agent 229: SSM optimization patterns" page,
// section 7), plus softplus(delta + bias), the D skip, the silu(z) gate and the
// final state.
//
// Kernel design (state-parallel, register-resident recurrence):
//  * The N states of one channel are split over TPC lanes of a warp (S = N/TPC
//    states per lane).  The states of a channel never interact except through
//    y = sum_n C_n h_n, so each lane runs its S recurrences sequentially over t
//    with no scan across time at all: one ex2 and four FP32 operations per
//    (t, n) -- the minimum the recurrence needs.  The per-lane partial sums of y
//    are reduced through shared memory once per block of TB time steps.
//  * A warp holds 32/TPC channels of one batch row; a CTA holds kWarps warps.
//    Channels never straddle a CTA's B/C group, so the B/C tile of a time block
//    is staged once in shared memory (fp32, [t][n]) and read by every channel.
//  * Per-(channel, t) work -- softplus, dt*u, the gate, the D skip, the
//    conversions and the 16-byte loads/stores -- is spread over the TPC lanes
//    of the channel (each lane owns TB/TPC consecutive steps), so it is done once.
//  * Global loads for block k+1 are issued before the recurrence of block k
//    (register double buffering), one __syncthreads per block.
//  * exp runs as ex2.approx with A pre-scaled by log2(e) once per lane.
//  * Time steps past L (the ragged last block) get dt = 0, i.e. dA = 1 and no
//    input, so the state is carried unchanged to last_state.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include "ssm_scan.h"

namespace ssm {

constexpr int kTB = 32;     // time steps per block
constexpr int kWarps = 4;   // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

struct FwdParams {
    const void* u;
    const void* delta;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const void* z;
    const float* bias;
    const float* h0;
    void* out;
    float* last_state;
    int* status;
    int64_t batch, dim, seqlen, nheads, ngroups;
    int softplus;
    int tiles_per_group;
};

// ----------------------------------------------------------------- helpers

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(x) = log(1 + e^x); above 20 it equals x to fp32 precision.
__device__ __forceinline__ float softplus_f32(float x) {
    return x > 20.f ? x : log1pf(expf(x));
}

__device__ __forceinline__ float silu_f32(float z) {
    return __fdividef(z, 1.f + ex2_approx(-z * kLog2e));
}

template <typename T> struct IO;
template <> struct IO<float> {
    static constexpr int kBytes = 4;
    __device__ static float get(const uint32_t* w, int e) { return __uint_as_float(w[e]); }
};
template <> struct IO<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    __device__ static float get(const uint32_t* w, int e) {
        uint32_t x = w[e >> 1];
        return __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
    }
};

// CNT consecutive elements of a row, starting at t, kept as raw 32-bit words.
template <typename T, int CNT>
struct Chunk {
    static constexpr int kWords = CNT * IO<T>::kBytes / 4;
    uint32_t w[kWords];
};

// VEC: the chunk is wholly in or out of range and its start is aligned to its
// size (up to 16 bytes) -> vector loads of 16 or 8 bytes.
template <typename T, int CNT, bool VEC>
__device__ __forceinline__ void load_chunk(Chunk<T, CNT>& c, const T* row, int64_t t, int64_t L) {
    constexpr int W = Chunk<T, CNT>::kWords;
    if constexpr (VEC) {
        static_assert(W % 2 == 0, "vector chunk must be a multiple of 8 bytes");
        if (t < L) {
            if constexpr (W % 4 == 0) {
                const uint4* p = reinterpret_cast<const uint4*>(row + t);
#pragma unroll
                for (int q = 0; q < W / 4; ++q) {
                    const uint4 v = __ldg(p + q);
                    c.w[4 * q + 0] = v.x; c.w[4 * q + 1] = v.y; c.w[4 * q + 2] = v.z; c.w[4 * q + 3] = v.w;
                }
            } else {
                const uint2* p = reinterpret_cast<const uint2*>(row + t);
#pragma unroll
                for (int q = 0; q < W / 2; ++q) {
                    const uint2 v = __ldg(p + q);
                    c.w[2 * q + 0] = v.x; c.w[2 * q + 1] = v.y;
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < W; ++q) c.w[q] = 0u;
        }
    } else {
        if constexpr (IO<T>::kBytes == 4) {
#pragma unroll
            for (int e = 0; e < CNT; ++e)
                c.w[e] = (t + e < L) ? __float_as_uint(__ldg(reinterpret_cast<const float*>(row) + t + e)) : 0u;
        } else {
            const unsigned short* r = reinterpret_cast<const unsigned short*>(row);
#pragma unroll
            for (int q = 0; q < CNT / 2; ++q) {
                const uint32_t lo = (t + 2 * q < L) ? (uint32_t)__ldg(r + t + 2 * q) : 0u;
                const uint32_t hi = (t + 2 * q + 1 < L) ? (uint32_t)__ldg(r + t + 2 * q + 1) : 0u;
                c.w[q] = lo | (hi << 16);
            }
        }
    }
}

// Store CNT consecutive outputs (rounded to nearest even for bf16).
template <typename T, int CNT, bool VEC>
__device__ __forceinline__ void store_chunk(T* row, int64_t t, int64_t L, const float (&v)[CNT]) {
    constexpr int W = CNT * IO<T>::kBytes / 4;
    uint32_t w[W];
    if constexpr (IO<T>::kBytes == 4) {
#pragma unroll
        for (int e = 0; e < CNT; ++e) w[e] = __float_as_uint(v[e]);
    } else {
#pragma unroll
        for (int q = 0; q < CNT / 2; ++q) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            w[q] = *reinterpret_cast<uint32_t*>(&b);
        }
    }
    if constexpr (VEC) {
        if (t < L) {
            if constexpr (W % 4 == 0) {
#pragma unroll
                for (int q = 0; q < W / 4; ++q)
                    reinterpret_cast<uint4*>(row + t)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            } else {
#pragma unroll
                for (int q = 0; q < W / 2; ++q) reinterpret_cast<uint2*>(row + t)[q] = make_uint2(w[2 * q], w[2 * q + 1]);
            }
        }
    } else {
        if constexpr (IO<T>::kBytes == 4) {
            uint32_t* r = reinterpret_cast<uint32_t*>(row);
#pragma unroll
            for (int e = 0; e < CNT; ++e)
                if (t + e < L) r[t + e] = w[e];
        } else {
            unsigned short* r = reinterpret_cast<unsigned short*>(row);
#pragma unroll
            for (int q = 0; q < CNT / 2; ++q) {
                if (t + 2 * q < L) r[t + 2 * q] = (unsigned short)(w[q] & 0xFFFFu);
                if (t + 2 * q + 1 < L) r[t + 2 * q + 1] = (unsigned short)(w[q] >> 16);
            }
        }
    }
}

// ------------------------------------------------------------ kernel config

template <typename T, int N>
struct Cfg {
    static constexpr int TPC = (N <= 8) ? 2 : (N == 16 ? 4 : 8);  // lanes per channel
    static constexpr int S = N / TPC;                               // states per lane
    static constexpr int CPW = 32 / TPC;                            // channels per warp
    static constexpr int CH = kWarps * CPW;                         // channels per CTA
    static constexpr int TPT = kTB / TPC;                           // steps per lane in pro/epilogue
    static constexpr int VE = 16 / IO<T>::kBytes;                   // elements per 16-byte B/C chunk
    static constexpr int BC_CHUNKS = 2 * N * (kTB / VE);            // B/C chunks per time block
    static constexpr int BC_PER_THREAD = (BC_CHUNKS + kThreads - 1) / kThreads;
    static constexpr int ROW = kTB + 4;                             // padded smem row (floats)
    // shared memory layout (floats)
    static constexpr int OFF_BC = 0;                                // [2 buf][2 B/C][kTB][N]
    static constexpr int SZ_BC = 2 * 2 * kTB * N;
    static constexpr int OFF_DT = OFF_BC + SZ_BC;                   // [kWarps][CPW][ROW] dt
    static constexpr int OFF_DTU = OFF_DT + kWarps * CPW * ROW;     // dt*u
    static constexpr int OFF_DA = OFF_DTU + kWarps * CPW * ROW;     // dA (scalar-A-per-head only)
    static constexpr int OFF_Y = OFF_DA + kWarps * CPW * ROW;       // [kWarps][CPW*TPC][ROW] partial y
    static constexpr int SMEM_FLOATS = OFF_Y + kWarps * CPW * TPC * ROW;
    static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
    static_assert(S % 4 == 0, "states per lane must be a multiple of 4");
    static_assert(TPT % 4 == 0, "steps per lane must be a multiple of 4");
    // the host takes the vector path only when L % 16 == 0, which keeps every
    // per-lane chunk wholly inside or outside a row only if chunks are <= 16
    static_assert(TPT <= 16 && VE <= 16, "chunks longer than 16 elements break the L % 16 rule");
};

// ------------------------------------------------------------------- kernel

template <typename T, int N, bool HEAD_A, bool VEC>
__global__ void __launch_bounds__(kThreads)
scan_fwd_kernel(const FwdParams p) {
    using C = Cfg<T, N>;
    constexpr int TPC = C::TPC, S = C::S, CPW = C::CPW, CH = C::CH, TPT = C::TPT, VE = C::VE, ROW = C::ROW;
    extern __shared__ __align__(16) float smem[];

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int cw = lane / TPC, j = lane % TPC;

    const int64_t Dm = p.dim, L = p.seqlen, H = p.nheads, G = p.ngroups;
    const int64_t Dg = Dm / G;
    const int64_t bg = blockIdx.x / p.tiles_per_group;
    const int64_t ti = blockIdx.x % p.tiles_per_group;
    const int64_t b = bg / G, g = bg % G;
    const int64_t ci = ti * CH + warp * CPW + cw;
    const bool valid = ci < Dg;
    const int64_t d = g * Dg + (valid ? ci : 0);
    const int64_t hd = d / (Dm / H);

    const T* u_row = reinterpret_cast<const T*>(p.u) + (b * Dm + d) * L;
    const T* z_row = p.z ? reinterpret_cast<const T*>(p.z) + (b * Dm + d) * L : nullptr;
    const T* dl_row = reinterpret_cast<const T*>(p.delta) + (b * H + hd) * L;
    T* out_row = reinterpret_cast<T*>(p.out) + (b * Dm + d) * L;
    const T* Bbase = reinterpret_cast<const T*>(p.B) + (b * G + g) * (int64_t)N * L;
    const T* Cbase = reinterpret_cast<const T*>(p.C) + (b * G + g) * (int64_t)N * L;

    // per-lane constants
    float a2[HEAD_A ? 1 : S];
    if constexpr (HEAD_A) {
        a2[0] = __ldg(p.A + hd) * kLog2e;
    } else {
#pragma unroll
        for (int s = 0; s < S; ++s) a2[s] = __ldg(p.A + d * N + j * S + s) * kLog2e;
    }
    const float Dd = p.D ? __ldg(p.D + d) : 0.f;
    const float bias = p.bias ? __ldg(p.bias + hd) : 0.f;
    float h[S];
#pragma unroll
    for (int s = 0; s < S; ++s) h[s] = p.h0 ? p.h0[(b * Dm + d) * N + j * S + s] : 0.f;

    float* sBC = smem + C::OFF_BC;
    float* sdt = smem + C::OFF_DT + (warp * CPW + cw) * ROW;
    float* sdtu = smem + C::OFF_DTU + (warp * CPW + cw) * ROW;
    float* sdA = smem + C::OFF_DA + (warp * CPW + cw) * ROW;
    float* sy_w = smem + C::OFF_Y + warp * CPW * TPC * ROW;

    // register prefetch buffers
    Chunk<T, TPT> pu, pdl, pz;
    Chunk<T, VE> pbc[C::BC_PER_THREAD];

    auto issue_loads = [&](int64_t t0) {
        const int64_t tl = t0 + j * TPT;
        if (valid) {
            load_chunk<T, TPT, VEC>(pu, u_row, tl, L);
            load_chunk<T, TPT, VEC>(pdl, dl_row, tl, L);
            if (z_row) load_chunk<T, TPT, VEC>(pz, z_row, tl, L);
        }
#pragma unroll
        for (int k = 0; k < C::BC_PER_THREAD; ++k) {
            const int c = tid + k * kThreads;
            if (c < C::BC_CHUNKS) {
                const int tc = c % (kTB / VE);
                const int n = (c / (kTB / VE)) % N;
                const int which = c / (N * (kTB / VE));
                const T* row = (which ? Cbase : Bbase) + (int64_t)n * L;
                load_chunk<T, VE, VEC>(pbc[k], row, t0 + tc * VE, L);
            }
        }
    };

    const int64_t nblk = (L + kTB - 1) / kTB;
    if (nblk > 0) issue_loads(0);

    for (int64_t k = 0; k < nblk; ++k) {
        const int64_t t0 = k * kTB;
        const int buf = (int)(k & 1);
        // -- prologue: dt, dt*u (and dA) for this lane's TPT steps
        float ucur[TPT], zcur[TPT];
#pragma unroll
        for (int i = 0; i < TPT; ++i) {
            const bool in = valid && (t0 + j * TPT + i < L);
            const float uv = in ? IO<T>::get(pu.w, i) : 0.f;
            const float x = (in ? IO<T>::get(pdl.w, i) : 0.f) + bias;
            float dt = p.softplus ? softplus_f32(x) : x;
            dt = in ? dt : 0.f;
            ucur[i] = uv;
            zcur[i] = (in && z_row) ? IO<T>::get(pz.w, i) : 0.f;
            sdt[j * TPT + i] = dt;
            sdtu[j * TPT + i] = dt * uv;
            if constexpr (HEAD_A) sdA[j * TPT + i] = ex2_approx(dt * a2[0]);
        }
        // -- stage the B/C tile (fp32, [t][n]) into buffer `buf`
        float* sB = sBC + buf * 2 * kTB * N;
#pragma unroll
        for (int q = 0; q < C::BC_PER_THREAD; ++q) {
            const int c = tid + q * kThreads;
            if (c < C::BC_CHUNKS) {
                const int tc = c % (kTB / VE);
                const int n = (c / (kTB / VE)) % N;
                const int which = c / (N * (kTB / VE));
                float* dst = sB + which * kTB * N;
#pragma unroll
                for (int e = 0; e < VE; ++e) dst[(tc * VE + e) * N + n] = IO<T>::get(pbc[q].w, e);
            }
        }
        __syncthreads();
        if (k + 1 < nblk) issue_loads(t0 + kTB);

        // -- the recurrence over this block
        const float* sBt = sB;
        const float* sCt = sB + kTB * N;
        float yp[kTB];
#pragma unroll
        for (int tq = 0; tq < kTB; tq += 4) {
            const float4 dt4 = *reinterpret_cast<const float4*>(sdt + tq);
            const float4 du4 = *reinterpret_cast<const float4*>(sdtu + tq);
            float4 da4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (HEAD_A) da4 = *reinterpret_cast<const float4*>(sdA + tq);
            const float dtv[4] = {dt4.x, dt4.y, dt4.z, dt4.w};
            const float duv[4] = {du4.x, du4.y, du4.z, du4.w};
            const float dav[4] = {da4.x, da4.y, da4.z, da4.w};
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int t = tq + tt;
                float Bv[S], Cv[S];
#pragma unroll
                for (int s4 = 0; s4 < S; s4 += 4) {
                    const float4 bb = *reinterpret_cast<const float4*>(sBt + t * N + j * S + s4);
                    const float4 cc = *reinterpret_cast<const float4*>(sCt + t * N + j * S + s4);
                    Bv[s4] = bb.x; Bv[s4 + 1] = bb.y; Bv[s4 + 2] = bb.z; Bv[s4 + 3] = bb.w;
                    Cv[s4] = cc.x; Cv[s4 + 1] = cc.y; Cv[s4 + 2] = cc.z; Cv[s4 + 3] = cc.w;
                }
                float y = 0.f;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const float dA = HEAD_A ? dav[tt] : ex2_approx(dtv[tt] * a2[HEAD_A ? 0 : s]);
                    h[s] = fmaf(dA, h[s], duv[tt] * Bv[s]);
                    y = fmaf(Cv[s], h[s], y);
                }
                yp[t] = y;
            }
        }
        // -- reduce the partial sums of y over the channel's TPC lanes
        float* myrow = sy_w + (cw * TPC + j) * ROW;
#pragma unroll
        for (int tq = 0; tq < kTB; tq += 4)
            *reinterpret_cast<float4*>(myrow + tq) = make_float4(yp[tq], yp[tq + 1], yp[tq + 2], yp[tq + 3]);
        __syncwarp();
        float o[TPT];
#pragma unroll
        for (int i = 0; i < TPT; ++i) o[i] = Dd * ucur[i];
#pragma unroll
        for (int jj = 0; jj < TPC; ++jj) {
            const float* r = sy_w + (cw * TPC + jj) * ROW + j * TPT;
#pragma unroll
            for (int i4 = 0; i4 < TPT; i4 += 4) {
                const float4 v = *reinterpret_cast<const float4*>(r + i4);
                o[i4] += v.x; o[i4 + 1] += v.y; o[i4 + 2] += v.z; o[i4 + 3] += v.w;
            }
        }
        if (z_row) {
#pragma unroll
            for (int i = 0; i < TPT; ++i) o[i] *= silu_f32(zcur[i]);
        }
        if (valid) store_chunk<T, TPT, VEC>(out_row, t0 + j * TPT, L, o);
        __syncwarp();
    }

    if (valid && p.last_state) {
        float* ls = p.last_state + (b * Dm + d) * N + j * S;
#pragma unroll
        for (int s = 0; s < S; ++s) ls[s] = h[s];
    }
}

// --------------------------------------------------------------- dispatch

using KernelFn = void (*)(const FwdParams);

struct Variant {
    KernelFn fn;
    int smem;
    int ch_per_cta;
    const char* name;
};

template <typename T, int N, bool HEAD_A, bool VEC>
Variant make_variant(const char* name) {
    return Variant{scan_fwd_kernel<T, N, HEAD_A, VEC>, Cfg<T, N>::SMEM_BYTES, Cfg<T, N>::CH, name};
}

// One function per (io dtype, N) translation unit; see fwd_*.cu.
#define SSM_DEFINE_PICK(T, TN, N)                                                                    \
    bool pick_##TN##_n##N(bool head, bool vec, Variant* v) {                                        \
        if (head)                                                                                   \
            *v = vec ? make_variant<T, N, true, true>("sp_" #TN "_n" #N "_head_vec")                \
                     : make_variant<T, N, true, false>("sp_" #TN "_n" #N "_head");                  \
        else                                                                                        \
            *v = vec ? make_variant<T, N, false, true>("sp_" #TN "_n" #N "_vec")                    \
                     : make_variant<T, N, false, false>("sp_" #TN "_n" #N);                         \
        return true;                                                                                \
    }

#define SSM_DECLARE_PICK(TN, N) bool pick_##TN##_n##N(bool head, bool vec, Variant* v);
SSM_DECLARE_PICK(bf16, 8)
SSM_DECLARE_PICK(bf16, 16)
SSM_DECLARE_PICK(bf16, 32)
SSM_DECLARE_PICK(bf16, 64)
SSM_DECLARE_PICK(bf16, 128)
SSM_DECLARE_PICK(f32, 8)
SSM_DECLARE_PICK(f32, 16)
SSM_DECLARE_PICK(f32, 32)
SSM_DECLARE_PICK(f32, 64)
SSM_DECLARE_PICK(f32, 128)

}  // namespace ssm
