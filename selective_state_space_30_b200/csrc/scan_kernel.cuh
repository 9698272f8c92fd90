#pragma once
// Selective-SSM (S6) forward scan kernel for B200 (sm_100a).
//
// What it computes is stated in include/ssm_scan.h: the recurrence of the
// Mamba "architecture-details" page (section "How S6 Works") with
// A_bar = exp(dt*A) (the "Agent 229: SSM optimization patterns" page, section 7),
// plus dt = softplus(delta + bias), the D skip, the silu(z) gate and the final state.
//
// Design (B200-first):
//
//  * State-parallel, register-resident recurrence.  The N states of a channel
//    are split over TPC lanes of a warp (S = N/TPC states per lane, S = 2 or 4
//    for N <= 16, 4 for N = 32, N/8 above); each lane runs its states
//    sequentially over t.  States only meet in
//    y = sum_n C_n h_n, so there is no scan across time inside a segment: one
//    ex2 per (t, n) plus four FP32 operations (issued as packed f32x2).
//  * Warp-specialised persistent CTAs, one per SM: a producer warp and W
//    consumer warps (W = 16, 8 or 4: four, two or one per SM sub-partition; ex2
//    issues per sub-partition and the kernel is latency-bound, so the most warps
//    that still give every SM a channel tile win).
//    - The producer takes work units -- (channel tile of W*CW channels, L
//      segment) -- from a global ticket counter in segment-major order, waits
//      (bounded) for the previous segment of the tile to publish its state,
//      loads the unit's parameters and incoming state into shared memory, and
//      streams each 32-step block of u, delta, z rows and B, C rows into a
//      STAGES-deep shared-memory ring with cp.async.bulk, completing on an
//      mbarrier.  It also publishes each finished segment's state (carry
//      buffer, then a release flag).  All global-memory latency sits in this
//      warp.
//    - Consumer warps only compute: wait for a full stage, run the block,
//      arrive on the stage's empty barrier.  No CTA-wide barrier.
//  * A unit's predecessor was ticketed earlier by a running producer, so the
//    chain always progresses; every wait is bounded and records
//    SSM_ERR_TIMEOUT in the workspace status instead of hanging.
//  * B and C rows sit in shared memory in transposed row order (state s of
//    lane group j at row s*TPC + j) with a 16-byte row pad, so the TPC lanes of
//    a channel read different banks.
//  * The per-(channel, t) work -- softplus, dt*u, the gate, the D skip -- is
//    spread over the TPC lanes of the channel (lane j owns steps
//    [j*TPT, (j+1)*TPT) of the block).  The per-lane partial sums of y are
//    reduce-scattered with shuffles per window of steps.
//  * softplus(x) = max(x,0) + log1p(2^(-|x| log2 e)) with one ex2 and a degree-7
//    polynomial for log1p(e)/e on [0, 1]: the Remez minimax fit of its relative
//    error, coefficients rounded to fp32 (1.9e-7 in exact arithmetic, 3.4e-7
//    for e*q(e) evaluated in fp32).
//  * Steps past L in the ragged last block get dt = 0 (dA = 1, no input) and
//    zeroed B, C, so the state reaches last_state unchanged.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ssm_scan.h"
#include "tcgen05.cuh"

namespace ssm {

constexpr int kTB = 32;      // time steps per block: the fp32 and tensor-memory kernels
constexpr int kTB16 = 64;    // time steps per block: the register kernel with bf16 I/O
constexpr int kSegAlign = 64;  // segment lengths are multiples of every block length
constexpr int kStages = 3;   // shared-memory ring depth (2 where 3 do not fit)
constexpr float kLog2e = 1.4426950408889634f;

// Device workspace owned by the plan (zeroed at plan creation; the last CTA of
// every launch puts the counters and flags back to zero).
struct WsHeader {
    unsigned ticket;  // next unit to hand out
    unsigned done;    // CTAs that have finished
    int status;       // kernel-side ssm_status_t (first error wins)
    unsigned inject;  // test hook: nonzero makes chained waits wait for a flag nobody sets
};

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
    WsHeader* ws;
    unsigned* flags;   // [n_tiles]: segments of the tile whose final state is published
    float* carry;      // [n_tiles][CT][N]
    int64_t batch, dim, seqlen, nheads, ngroups;
    int softplus;
    int tiles_per_group;
    int n_tiles;
    int n_seg;
    int seg_len;       // a multiple of the kernel's block length
    unsigned n_units;
    unsigned n_ctas;
    unsigned spin_limit;
    int delta_rows;    // rows of the delta box: CT (S6 layout) or the heads a tile can touch
    // optional (register kernel): the state entering every 8-step window, for the backward,
    // at ckpt[((b * dim + d) * ckpt_wins + t / 8) * N + n]; nullptr: not stored
    float* ckpt;
    int64_t ckpt_wins;
};

// The five 2-D tensor maps (time x rows) the producer loads boxes through.
struct TensorMaps {
    CUtensorMap u, delta, z, B, C;
};

// ----------------------------------------------------------------- helpers

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// packed fp32 pairs (sm_100 f32x2 instructions)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

// softplus(x) = max(x,0) + e*q(e), e = 2^(-|x| log2 e) in (0, 1], q the degree-7
// polynomial of least maximum relative error for log1p(e)/e on [0, 1] (a Remez
// exchange in fp64, then each coefficient rounded to fp32; e*q(e) evaluated in
// fp32 stays within 3.4e-7 of log1p(e)); coefficients from the highest degree down.
__device__ constexpr float kSoftplusQ[8] = {-0.008539234288036823f, 0.044089723378419876f, -0.10768184065818787f,
                                            0.17745250463485718f,   -0.2449546605348587f,  0.33275479078292847f,
                                            -0.4999740421772003f,   0.9999998211860657f};

// softplus on a pair
__device__ __forceinline__ float2 softplus2(float2 x) {
    const float2 a = mul2(make_float2(fabsf(x.x), fabsf(x.y)), dup2(-kLog2e));
    const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
    float2 q = dup2(kSoftplusQ[0]);
#pragma unroll
    for (int i = 1; i < 8; ++i) q = fma2(q, e, dup2(kSoftplusQ[i]));
    return fma2(e, q, make_float2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)));
}

__device__ __forceinline__ float softplus1(float x) {
    const float e = ex2_approx(fabsf(x) * -kLog2e);
    float q = kSoftplusQ[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) q = fmaf(q, e, kSoftplusQ[i]);
    return fmaf(e, q, fmaxf(x, 0.f));
}

// silu(z) = z / (1 + e^-z) on a pair, and on one value
__device__ __forceinline__ float2 silu2(float2 z) {
    const float2 a = mul2(z, dup2(-kLog2e));
    const float2 d = add2(make_float2(ex2_approx(a.x), ex2_approx(a.y)), dup2(1.f));
    return mul2(z, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

__device__ __forceinline__ float silu1(float z) { return z * rcp_approx(ex2_approx(z * -kLog2e) + 1.f); }

// a global store that only lanes with c set perform (a predicated store, no branch)
__device__ __forceinline__ void st_global_if(float* p, float v, bool c) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.f32 [%0], %1;\n\t}" ::"l"(p), "f"(v),
                 "r"((int)c));
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename T> struct IO;
template <> struct IO<float> {
    static constexpr int kBytes = 4;
    __device__ static float get(const uint32_t* w, int e) { return __uint_as_float(w[e]); }
    // elements e, e+1 (e even)
    __device__ static float2 get2(const uint32_t* w, int e) {
        return make_float2(__uint_as_float(w[e]), __uint_as_float(w[e + 1]));
    }
};
template <> struct IO<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    __device__ static float get(const uint32_t* w, int e) {
        const uint32_t x = w[e >> 1];
        return __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
    }
    __device__ static float2 get2(const uint32_t* w, int e) {
        const uint32_t x = w[e >> 1];
        return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
    }
};

// CNT consecutive elements of a row held as raw 32-bit words.
template <typename T, int CNT>
struct Chunk {
    static constexpr int kWords = (CNT * IO<T>::kBytes + 3) / 4;
    uint32_t w[kWords];
};

template <typename T, int CNT, bool VEC>
__device__ __forceinline__ void store_chunk(T* row, int64_t t, int64_t L, const float (&v)[CNT]) {
    constexpr int W = (CNT * IO<T>::kBytes + 3) / 4;
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
            } else if constexpr (W % 2 == 0) {
#pragma unroll
                for (int q = 0; q < W / 2; ++q) reinterpret_cast<uint2*>(row + t)[q] = make_uint2(w[2 * q], w[2 * q + 1]);
            } else {
                reinterpret_cast<uint32_t*>(row + t)[0] = w[0];
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
            for (int e = 0; e < CNT; ++e)
                if (t + e < L) r[t + e] = (unsigned short)(w[e >> 1] >> (16 * (e & 1)));
        }
    }
}

// Reduce-scatter of a window of WT partial sums over the TPC lanes of a channel
// group (lane bits below TPC): each step halves the values a lane holds, then
// any remaining lane bits are summed by butterfly.  On return the lane holds the
// totals for window positions [off, off + max(1, WT/TPC)).
template <int WT, int TPC>
__device__ __forceinline__ void window_reduce(float (&a)[WT], int j, int& off) {
    off = 0;
#pragma unroll
    for (int s = 0; (TPC >> (s + 1)) >= 1; ++s) {
        const int m = TPC >> (s + 1);
        if ((WT >> s) >= 2) {
            const int half = WT >> (s + 1);
            const bool up = (j & m) != 0;
            float recv[WT / 2 > 0 ? WT / 2 : 1];
#pragma unroll
            for (int i = 0; i < half; ++i) recv[i] = __shfl_xor_sync(0xffffffffu, up ? a[i] : a[half + i], m);
            if (half % 2 == 0) {
#pragma unroll
                for (int i = 0; i < half; i += 2) {
                    const float2 k2 = up ? make_float2(a[half + i], a[half + i + 1]) : make_float2(a[i], a[i + 1]);
                    const float2 r2 = add2(k2, make_float2(recv[i], recv[i + 1]));
                    a[i] = r2.x;
                    a[i + 1] = r2.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < half; ++i) a[i] = (up ? a[half + i] : a[i]) + recv[i];
            }
            off += up ? half : 0;
        } else {
            a[0] += __shfl_xor_sync(0xffffffffu, a[0], m);
        }
    }
}

// ------------------------------------------------------ barriers and copies

__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
// non-blocking probe of a phase
__device__ __forceinline__ bool mbar_test(uint64_t* b, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}
// probe that may suspend the thread for a short, hardware-bounded time
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for a phase: false (and SSM_ERR_TIMEOUT recorded) after budget_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity, uint64_t budget_ns, int* status) {
    if (mbar_try(b, parity)) return true;
    const uint64_t t0 = now_ns();
    while (true) {
        if (mbar_try(b, parity)) return true;
        if (now_ns() - t0 > budget_ns) {
            atomicCAS(status, SSM_OK, SSM_ERR_TIMEOUT);
            return false;
        }
    }
}
// A float range src[i0, i0 + cnt) of an array of `total` elements, planned as one
// bulk copy of its 16-byte aligned superset when that superset stays inside the
// array (else: element copies).  off = position of i0 in the destination.
struct RangeCopy {
    int64_t start;   // first element copied
    int n;           // elements copied
    int off;         // i0 - start
    bool bulk;
};
__device__ __forceinline__ RangeCopy plan_range(const float* src, int64_t i0, int cnt, int64_t total) {
    RangeCopy r;
    const int64_t s4 = i0 & ~(int64_t)3;
    const int64_t e4 = (i0 + cnt + 3) & ~(int64_t)3;
    const bool aligned_base = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    r.bulk = aligned_base && cnt > 0 && e4 <= total;
    r.start = r.bulk ? s4 : i0;
    r.n = r.bulk ? (int)(e4 - s4) : cnt;
    r.off = (int)(i0 - r.start);
    return r;
}

// warp-uniform decision taken by lane 0
__device__ __forceinline__ bool lane0_says(bool v) { return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0; }

// Debug builds (compiled with SSM_DEBUG): an index outside its buffer records
// SSM_ERR_BOUNDS in the status word (first error wins) and the access is skipped; no
// trap.  Release builds compile the checks away.
__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
#ifdef SSM_DEBUG
    if (!ok) atomicCAS(status, SSM_OK, SSM_ERR_BOUNDS);
    return ok;
#else
    (void)ok;
    (void)status;
    return true;
#endif
}

__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// ------------------------------------------------------------ kernel config

template <typename T, int N, int W, bool HEAD_A, int SPL>
struct Cfg {
    using Elem = T;
    static constexpr bool kHeadA = HEAD_A;
    static constexpr int kN = N;
    static constexpr int ESZ = IO<T>::kBytes;
    // steps per block: 64 for bf16 I/O (a block's rows are 128 bytes either way, the
    // widest hardware swizzle; the longer block halves the per-block work), 32 for fp32
    static constexpr int TB = ESZ == 2 ? kTB16 : kTB;
    static constexpr int S = SPL;                          // states per lane
    static constexpr int TPC = N / S;                      // lanes per channel (2, 4 or 8)
    static constexpr int GW = 32 / TPC;                    // channels per consumer warp
    static constexpr int CT = W * GW;                      // channels per tile
    static constexpr int TPT = TB / TPC;                   // steps per lane in prologue / epilogue
    static constexpr int WT = (ESZ == 4 || S >= 16) ? 4 : 8;  // steps per B/C register window
    static constexpr int RB = TB * ESZ;                    // bytes of one block row
    static constexpr int ROW = TB + 4;                     // per-warp float rows (padded)
    static constexpr int NA = HEAD_A ? 1 : S;
    // one ring stage (1024-byte aligned): B box | C box (N rows each, hardware
    // swizzled) | u box | delta box | z box (CT rows each) | header
    static constexpr int OFF_BC = 0;
    static constexpr int OFF_IN = OFF_BC + 2 * N * RB;
    static constexpr int OFF_HDR = OFF_IN + 3 * CT * RB;
    static constexpr int STAGE = (OFF_HDR + 64 + 1023) / 1024 * 1024;
    // unit parameter slot (floats): A, D, bias (each with room for a 16-byte
    // aligned superset of the needed range) and the incoming state
    static constexpr int P_A = 0;
    static constexpr int P_D = P_A + (HEAD_A ? CT : CT * N) + 8;
    static constexpr int P_BIAS = P_D + CT + 8;
    static constexpr int P_H = P_BIAS + CT + 8;
    static constexpr int PSLOT = P_H + CT * N;
    static constexpr int CSLOT = CT * N;                   // outgoing state slot (floats)
    // per consumer warp (floats): dt, dt*u, (dA), reduced y
    static constexpr int W_DT = 0;
    static constexpr int W_DU = GW * ROW;
    static constexpr int W_DA = 2 * GW * ROW;
    static constexpr int W_Y = (HEAD_A ? 3 : 2) * GW * ROW;
    // Per-lane y rows (up to 8 consumer warps, where they fit): each lane writes its
    // partial sums of y over its S states to a row of its own, and the epilogue adds
    // the TPC rows of a channel, so the recurrence has no cross-lane reduction.  In
    // lane j's row, the TPT columns the epilogue of lane j reads are shifted by
    // YSH(j) 16-byte groups, which puts the eight lanes of each shared-memory phase in
    // different banks both when they write (same column, rows 17 groups apart) and when
    // they read (the rows of one channel, their own columns).
    static constexpr bool YLANE = W <= 8 && WT == 8 && TPT % 4 == 0;
    static constexpr int YSH_MAX = TPC == 8 ? 1 : TPC - 1;
    static constexpr int YROW = TB + 4 * YSH_MAX;
    // Per-lane-pair y rows (16 warps, 8 lanes per channel, 64-step blocks): the
    // recurrence does the first round of the reduction (lanes j and j^4 swap window
    // halves) and writes the pair's sums to row j&3, the lower halves from column 0 and
    // the upper halves from column YHALF; the epilogue adds the 4 rows.  A row is 18
    // 16-byte groups (2 mod 8) and YHALF 9 groups (1 mod 8), so the eight lanes of a
    // phase hit different banks on both sides.
    static constexpr bool YPART = !YLANE && W == 16 && TPC == 8 && WT == 8 && TB == 64;
    static constexpr int YPROW = 72, YHALF = 36;
    static constexpr int WARP_F = W_Y + (YLANE ? 32 * YROW : YPART ? GW * 4 * YPROW : GW * ROW);
    __device__ static constexpr int ysh(int jl) { return TPC == 8 ? jl >> 2 : jl; }
    // shared memory map (bytes)
    static constexpr int OFF_STAGES = 1024;                // barriers live below
    static constexpr int REST = 2 * PSLOT * 4 + 2 * CSLOT * 4 + W * WARP_F * 4;
    static constexpr int STG = OFF_STAGES + kStages * STAGE + REST <= 227 * 1024 ? kStages : 2;
    static constexpr int OFF_PSLOT = OFF_STAGES + STG * STAGE;
    static constexpr int OFF_CSLOT = OFF_PSLOT + 2 * PSLOT * 4;
    static constexpr int OFF_WARP = OFF_CSLOT + 2 * CSLOT * 4;
    static constexpr int SMEM = OFF_WARP + W * WARP_F * 4;
    static constexpr int THREADS = 32 * (W + 1);
    // the layout compiles: lanes per channel, 4 .. 16 steps per lane, the shared-memory budget
    static constexpr bool kFits = TPC >= 2 && TPC <= 8 && TPT % 4 == 0 && TPT <= 16 && SMEM <= 227 * 1024;
    static_assert(S % 2 == 0 && N % S == 0, "lane split");
    static_assert(STAGE % 16 == 0 && (PSLOT * 4) % 16 == 0 && (WARP_F * 4) % 16 == 0, "16-byte aligned smem");
    static_assert(2 * kStages + 6 <= 128, "barriers fit below OFF_STAGES");
    static_assert(RB == 64 || (N * RB) % 1024 == 0, "C box keeps the swizzle phase");
};

// Byte offset of element t of row r inside a B or C box of TB steps, as the
// tensor-map swizzle lays it out: 16-byte chunks XORed with row bits (64-byte rows:
// bits 1-2 of the row; 128-byte rows: bits 0-2).
template <int ESZ, int TB>
__device__ __forceinline__ int bc_off(int r, int t) {
    constexpr int RB = TB * ESZ;
    const int byte = t * ESZ;
    const int swz = RB == 64 ? ((r >> 1) & 3) : (r & 7);
    return r * RB + ((((byte >> 4) ^ swz) & (RB / 16 - 1)) << 4) + (byte & 15);
}

// barrier slots
enum { BAR_FULL = 0, BAR_EMPTY = kStages, BAR_PEMPTY = 2 * kStages, BAR_CFULL = 2 * kStages + 2,
       BAR_CEMPTY = 2 * kStages + 4 };

// per-block header written by the producer into its ring stage
struct BlockHdr {
    int64_t t0, t1;     // first step of the block; end of the unit's range
    int b, g, ci0;      // batch row, group, first channel-in-group of the tile
    int tile, seg;
    int flags;          // kFirst | kLast | kFinalSeg | kEnd
    int pslot;          // parameter slot of the unit
    int cseq;           // outgoing-state sequence number (last block of a non-final segment)
    int oa, od, ob;     // where element 0 of the tile's A, D, bias ranges sit in their slot regions
    int pad;
};
constexpr int kFirst = 1, kLast = 2, kFinalSeg = 4, kEnd = 8;
static_assert(sizeof(BlockHdr) <= 64, "header fits its slot");

// ------------------------------------------------------------------ producer

// The barriers a producer drives: fill[NST] (the stage's copies landed: TMA bytes or
// the producer's own element copies), empty[NST] (the consumers are done with the
// stage), and the two-slot handshakes of the unit parameters (pempty) and of the
// outgoing segment states (cfull, cempty).
struct ProducerBars {
    uint64_t *fill, *empty, *pempty, *cfull, *cempty;
};

// The producer warp of a scan kernel (Cf: the kernel's shared-memory map).  It takes
// work units -- (channel tile, L segment) -- from the global ticket counter in
// segment-major order, waits (bounded) for the previous segment of the tile to
// publish its state, loads the unit's parameters and incoming state into a
// parameter slot, streams each 32-step block of u, delta, z rows and B, C rows into
// the stage ring (five 2-D TMA boxes, or guarded element copies where a tensor map
// cannot describe the rows), and publishes every finished segment's state (carry
// buffer, then a release flag).  Every loop decision is taken by lane 0 and
// broadcast, so the warp never diverges.
template <class Cf, bool VEC>
__device__ __forceinline__ void produce(const FwdParams& p, const TensorMaps& tm, unsigned char* smem,
                                        const ProducerBars& br, int lane, uint64_t budget, int* status) {
    using T = typename Cf::Elem;
    constexpr bool HEAD_A = Cf::kHeadA;
    constexpr int N = Cf::kN, CT = Cf::CT, ESZ = Cf::ESZ, RB = Cf::RB, NST = Cf::STG, TB = Cf::TB;
    const int64_t Dm = p.dim, L = p.seqlen, H = p.nheads, G = p.ngroups;
    const int64_t Dg = Dm / G, P = Dm / H;
    unsigned fill = 0;          // blocks produced
    unsigned ucount = 0;        // units started
    unsigned pub_head = 0, pub_tail = 0;
    int pub_tile[2] = {0, 0}, pub_seg[2] = {0, 0};
    bool alive = true;

    // publish the outgoing state of finished segments (oldest first); every
    // loop decision below is taken by lane 0 and broadcast, so the warp never diverges
    auto service = [&](bool block) {
        while (pub_head < pub_tail) {
            const int slot = pub_head & 1;
            const unsigned par = (pub_head >> 1) & 1;
            bool ready;
            if (block) ready = lane0_says(lane == 0 ? mbar_wait(br.cfull + slot, par, budget, status) : false);
            else ready = lane0_says(lane == 0 ? mbar_test(br.cfull + slot, par) : false);
            if (!ready) {
                if (block) alive = false;
                return;
            }
            __syncwarp();  // order the other lanes' reads after lane 0's acquire
            const float* cs = reinterpret_cast<const float*>(smem + Cf::OFF_CSLOT) + slot * Cf::CSLOT;
            const int tile = slot ? pub_tile[1] : pub_tile[0];
            const int seg = slot ? pub_seg[1] : pub_seg[0];
            float* dst = p.carry + (int64_t)tile * CT * N;
            if (in_bounds(tile >= 0 && tile < p.n_tiles, status))
                for (int i = lane; i < CT * N; i += 32) __stcg(dst + i, cs[i]);
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                st_release(p.flags + tile, (unsigned)seg + 1u);
                mbar_arrive(br.cempty + slot);
            }
            ++pub_head;
        }
    };

    // wait for a free ring stage, publishing finished segments meanwhile
    auto acquire_stage = [&](unsigned f) -> bool {
        if (f < NST) return true;
        uint64_t* e = br.empty + f % NST;
        const unsigned par = ((f / NST) - 1) & 1;
        // the suspending try_wait keeps the producer off the issue slots it shares
        // with the consumer warps of its SM sub-partition
        if (lane0_says(lane == 0 ? mbar_try(e, par) : false)) { __syncwarp(); return true; }
        const uint64_t t0 = now_ns();
        while (!lane0_says(lane == 0 ? mbar_try(e, par) : false)) {
            service(false);
            if (lane0_says(lane == 0 ? now_ns() - t0 > budget : false)) {
                if (lane == 0) atomicCAS(status, SSM_OK, SSM_ERR_TIMEOUT);
                return false;
            }
            __nanosleep(256);
        }
        __syncwarp();
        return true;
    };

    while (alive) {
        unsigned tk = 0;
        if (lane == 0) tk = atomicAdd(&p.ws->ticket, 1u);
        tk = __shfl_sync(0xffffffffu, tk, 0);
        if (tk >= p.n_units) break;
        const int seg = (int)(tk / (unsigned)p.n_tiles);
        const int tile = (int)(tk % (unsigned)p.n_tiles);
        const int bg = tile / p.tiles_per_group, ti = tile % p.tiles_per_group;
        const int64_t b = bg / G, g = bg % G, ci0 = (int64_t)ti * CT;
        const int64_t t0u = (int64_t)seg * p.seg_len;
        const int64_t t1u = t0u + p.seg_len < L ? t0u + p.seg_len : L;
        const int nblk = L > 0 ? (int)((t1u - t0u + TB - 1) / TB) : 1;
        const bool final_seg = seg + 1 >= p.n_seg;
        const int pslot = ucount & 1;

        // the parameter slot must have been read by the consumers (unit ucount-2)
        if (ucount >= 2) {
            const unsigned par = ((ucount >> 1) - 1) & 1;
            const uint64_t tw = now_ns();
            while (!lane0_says(lane == 0 ? mbar_try(br.pempty + pslot, par) : false)) {
                service(false);
                __nanosleep(256);
                if (lane0_says(lane == 0 ? now_ns() - tw > budget : false)) {
                    if (lane == 0) atomicCAS(status, SSM_OK, SSM_ERR_TIMEOUT);
                    alive = false;
                    break;
                }
            }
            if (!alive) break;
            __syncwarp();
        }
        // the previous segment of the tile must have published its state
        bool carry_ok = true;
        if (seg > 0) {
            const unsigned need = (unsigned)seg + (p.ws->inject ? 0x40000000u : 0u);
            const uint64_t tw = now_ns();
            while (true) {
                // 0 = ready, 1 = keep waiting, 2 = give up
                int outcome = 1;
                if (lane == 0) {
                    if (ld_acquire(p.flags + tile) >= need) outcome = 0;
                    else if (*reinterpret_cast<volatile int*>(status) != SSM_OK) outcome = 2;
                    else if (now_ns() - tw > budget) {
                        atomicCAS(status, SSM_OK, SSM_ERR_TIMEOUT);
                        outcome = 2;
                    }
                }
                outcome = __shfl_sync(0xffffffffu, outcome, 0);
                if (outcome == 0) break;
                if (outcome == 2) { carry_ok = false; break; }
                service(false);
                __nanosleep(200);
            }
            __syncwarp();
        }
        // parameters and incoming state of the unit -> parameter slot, by bulk
        // copies that complete on the unit's first-block barrier (element copies
        // only where a range is not 16-byte aligned inside its array)
        float* ps = reinterpret_cast<float*>(smem + Cf::OFF_PSLOT) + pslot * Cf::PSLOT;
        const int nvalid_u = (int)(Dg - ci0 < CT ? Dg - ci0 : CT);
        const int64_t d0 = g * Dg + ci0;
        const int64_t h_lo = d0 / P, h_hi = (d0 + nvalid_u - 1) / P;
        const RangeCopy rA = HEAD_A ? plan_range(p.A, h_lo, (int)(h_hi - h_lo + 1), H)
                                    : plan_range(p.A, d0 * N, nvalid_u * N, Dm * N);
        const RangeCopy rD = plan_range(p.D, d0, nvalid_u, Dm);
        const RangeCopy rB = plan_range(p.bias, h_lo, (int)(h_hi - h_lo + 1), H);
        const float* hsrc = seg == 0 ? (p.h0 ? p.h0 + (b * Dm + d0) * N : nullptr)
                                     : (carry_ok ? p.carry + (int64_t)tile * CT * N : nullptr);
        const int hcnt = seg == 0 ? nvalid_u * N : CT * N;
        const bool hbulk = hsrc && (reinterpret_cast<uintptr_t>(hsrc) & 15u) == 0 && (hcnt % 4) == 0;
        unsigned ptx = (rA.bulk ? rA.n * 4u : 0u) + (p.D && rD.bulk ? rD.n * 4u : 0u) +
                       (p.bias && rB.bulk ? rB.n * 4u : 0u) + (hbulk ? hcnt * 4u : 0u);
        // element copies and zero fills (generic stores, published by the first block's arrive)
        if (!rA.bulk)
            for (int i = lane; i < rA.n; i += 32) ps[Cf::P_A + i] = __ldg(p.A + rA.start + i);
        if (!p.D) for (int i = lane; i < CT; i += 32) ps[Cf::P_D + i] = 0.f;
        else if (!rD.bulk) for (int i = lane; i < rD.n; i += 32) ps[Cf::P_D + i] = __ldg(p.D + rD.start + i);
        if (!p.bias) for (int i = lane; i < CT + 8; i += 32) ps[Cf::P_BIAS + i] = 0.f;
        else if (!rB.bulk) for (int i = lane; i < rB.n; i += 32) ps[Cf::P_BIAS + i] = __ldg(p.bias + rB.start + i);
        if (!hsrc) for (int i = lane; i < CT * N; i += 32) ps[Cf::P_H + i] = 0.f;
        else if (!hbulk) for (int i = lane; i < hcnt; i += 32) ps[Cf::P_H + i] = __ldcg(hsrc + i);
        if (hbulk && seg > 0) asm volatile("fence.proxy.async.global;" ::: "memory");
        int cseq = 0;
        if (!final_seg) {
            // at most two outgoing states in flight: publish the oldest first
            while (pub_tail - pub_head >= 2 && alive) service(true);
            cseq = (int)pub_tail;
            if (pub_tail & 1) { pub_tile[1] = tile; pub_seg[1] = seg; }
            else { pub_tile[0] = tile; pub_seg[0] = seg; }
            ++pub_tail;
        }
        __syncwarp();
        // stream the unit's blocks
        for (int kb = 0; kb < nblk && alive; ++kb, ++fill) {
            if (!acquire_stage(fill)) { alive = false; break; }
            const int st = fill % NST;
            unsigned char* sb = smem + Cf::OFF_STAGES + st * Cf::STAGE;
            uint64_t* full = br.fill + st;
            const int64_t t0 = t0u + (int64_t)kb * TB;
            const int64_t nv = L - t0 < TB ? (L - t0 > 0 ? L - t0 : 0) : TB;  // valid steps in the block
            int nvalid = (int)(Dg - ci0 < CT ? Dg - ci0 : CT);
            if (lane == 0) {
                BlockHdr* hd = reinterpret_cast<BlockHdr*>(sb + Cf::OFF_HDR);
                hd->b = (int)b; hd->g = (int)g; hd->ci0 = (int)ci0; hd->t0 = t0; hd->t1 = t1u;
                hd->tile = tile; hd->seg = seg;
                hd->flags = (kb == 0 ? kFirst : 0) | (kb == nblk - 1 ? kLast : 0) | (final_seg ? kFinalSeg : 0);
                hd->pslot = pslot; hd->cseq = cseq;
                hd->oa = rA.off; hd->od = rD.off; hd->ob = rB.off;
            }
            const unsigned extra_tx = kb == 0 ? ptx : 0u;
            // the unit's parameter bulk copies ride on its first block's barrier
            auto issue_params = [&]() {
                if (kb != 0 || lane != 0) return;
                if (rA.bulk) bulk_g2s(ps + Cf::P_A, p.A + rA.start, rA.n * 4u, full);
                if (p.D && rD.bulk) bulk_g2s(ps + Cf::P_D, p.D + rD.start, rD.n * 4u, full);
                if (p.bias && rB.bulk) bulk_g2s(ps + Cf::P_BIAS, p.bias + rB.start, rB.n * 4u, full);
                if (hbulk) bulk_g2s(ps + Cf::P_H, hsrc, hcnt * 4u, full);
            };
            const int ntens = p.z ? 3 : 2;
            const int64_t d0b = g * Dg + ci0;          // first channel of the tile
            const int64_t hrow0 = HEAD_A ? d0b / P : d0b;  // first delta row of the tile
            if (VEC) {
                // five 2-D boxes; the tensor maps zero-fill whatever lies past L or past the last row
                const unsigned bytes = (unsigned)RB * (unsigned)(2 * N + CT + p.delta_rows + (ntens == 3 ? CT : 0));
                const bool coords_ok = t0 >= 0 && t0 < L && (b * G + g) * N + N <= p.batch * G * N &&
                                       b * Dm + d0b < p.batch * Dm && b * H + hrow0 < p.batch * H;
                if (lane == 0 && !in_bounds(coords_ok, status)) {
                    mbar_arrive_tx(full, extra_tx);
                } else if (lane == 0) {
                    mbar_arrive_tx(full, bytes + extra_tx);
                    const int x = (int)t0;
                    tma_2d(sb + Cf::OFF_BC, &tm.B, x, (int)((b * G + g) * N), full);
                    tma_2d(sb + Cf::OFF_BC + N * RB, &tm.C, x, (int)((b * G + g) * N), full);
                    tma_2d(sb + Cf::OFF_IN, &tm.u, x, (int)(b * Dm + d0b), full);
                    tma_2d(sb + Cf::OFF_IN + CT * RB, &tm.delta, x, (int)(b * H + hrow0), full);
                    if (ntens == 3) tma_2d(sb + Cf::OFF_IN + 2 * CT * RB, &tm.z, x, (int)(b * Dm + d0b), full);
                }
                __syncwarp();
                issue_params();
            } else {
                // guarded element copies into the same layout (unaligned rows, ragged tails)
                const T* Bb = reinterpret_cast<const T*>(p.B) + (b * G + g) * (int64_t)N * L;
                const T* Cb = reinterpret_cast<const T*>(p.C) + (b * G + g) * (int64_t)N * L;
                for (int e = lane; e < 2 * N * TB; e += 32) {
                    const int r = e / TB, tt = e % TB;
                    const int w = r / N, n = r % N;
                    const T* src = (w ? Cb : Bb) + (int64_t)n * L;
                    *reinterpret_cast<T*>(sb + Cf::OFF_BC + w * N * RB + bc_off<ESZ, TB>(n, tt)) =
                        tt < nv ? src[t0 + tt] : T(0.f);
                }
                for (int e = lane; e < ntens * CT * TB; e += 32) {
                    const int r = e / TB, tt = e % TB;
                    const int w = r / CT, lcr = r % CT;
                    const T* src = nullptr;
                    if (w == 1) {
                        const int64_t hr = hrow0 + lcr;
                        if (lcr < p.delta_rows && hr < H) src = reinterpret_cast<const T*>(p.delta) + (b * H + hr) * L;
                    } else if (lcr < nvalid) {
                        src = reinterpret_cast<const T*>(w == 0 ? p.u : p.z) + (b * Dm + d0b + lcr) * L;
                    }
                    *reinterpret_cast<T*>(sb + Cf::OFF_IN + (w * CT + lcr) * RB + tt * ESZ) =
                        (src && tt < nv) ? src[t0 + tt] : T(0.f);
                }
                // generic stores made visible to the async proxy (tensor cores may read the boxes)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    if (extra_tx) mbar_arrive_tx(full, extra_tx);
                    else mbar_arrive(full);
                }
                __syncwarp();
                issue_params();
            }
            service(false);
        }
        ++ucount;
    }
    // end-of-work marker for the consumers
    if (acquire_stage(fill)) {
        const int st = fill % NST;
        if (lane == 0) {
            reinterpret_cast<BlockHdr*>(smem + Cf::OFF_STAGES + st * Cf::STAGE + Cf::OFF_HDR)->flags = kEnd;
            mbar_arrive(br.fill + st);
        }
        ++fill;
    }
    while (pub_head < pub_tail && alive) service(true);
    // the last CTA to finish resets the counters and flags for the next launch
    unsigned last = 0;
    if (lane == 0) {
        __threadfence();
        last = atomicAdd(&p.ws->done, 1u) == p.n_ctas - 1u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
        __threadfence();
        for (int i = lane; i < p.n_tiles; i += 32) p.flags[i] = 0u;
        if (lane == 0) {
            p.ws->ticket = 0u;
            p.ws->done = 0u;
        }
        __threadfence();
    }
}

// ------------------------------------------------------------------- kernel

// CKPT: also store the state entering every 8-step window (p.ckpt, for the backward)
template <typename T, int N, int W, bool HEAD_A, int SPL, bool VEC, bool CKPT>
__global__ void __launch_bounds__(Cfg<T, N, W, HEAD_A, SPL>::THREADS, 1)
scan_fwd_kernel(const FwdParams p, const __grid_constant__ TensorMaps tm) {
    using Cf = Cfg<T, N, W, HEAD_A, SPL>;
    constexpr int S = Cf::S, TPC = Cf::TPC, GW = Cf::GW, CT = Cf::CT, TPT = Cf::TPT, WT = Cf::WT;
    constexpr int ROW = Cf::ROW, NA = Cf::NA, ESZ = Cf::ESZ, RB = Cf::RB, TB = Cf::TB;
    constexpr int NST = Cf::STG;  // ring stages
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Dm = p.dim, L = p.seqlen, H = p.nheads, G = p.ngroups;
    const int64_t Dg = Dm / G, P = Dm / H;
    int* status = &p.ws->status;
    const uint64_t budget = (uint64_t)p.spin_limit * 256ull;  // ns

    // the swizzle of the B and C boxes assumes a 1024-byte aligned base
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(status, SSM_OK, SSM_ERR_BOUNDS);
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bars + BAR_FULL + s, 1);
            mbar_init(bars + BAR_EMPTY + s, W);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bars + BAR_PEMPTY + s, W);
            mbar_init(bars + BAR_CFULL + s, W);
            mbar_init(bars + BAR_CEMPTY + s, 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == W) {
        // ============================================================ producer
        produce<Cf, VEC>(p, tm, smem,
                         ProducerBars{bars + BAR_FULL, bars + BAR_EMPTY, bars + BAR_PEMPTY, bars + BAR_CFULL,
                                      bars + BAR_CEMPTY},
                         lane, budget, status);
        return;
    }

    // ================================================================ consumers
    const int cg = lane / TPC, j = lane % TPC;
    const int lc = warp * GW + cg;   // channel of the lane within the tile
    float* wf = reinterpret_cast<float*>(smem + Cf::OFF_WARP) + warp * Cf::WARP_F;
    float* rdt = wf + Cf::W_DT + cg * ROW;
    float* rdu = wf + Cf::W_DU + cg * ROW;
    float* rda = wf + Cf::W_DA + cg * ROW;
    float* ry = wf + Cf::W_Y + cg * (Cf::YLANE ? TPC * Cf::YROW : Cf::YPART ? 4 * Cf::YPROW : ROW);
    // this lane's states are n = s*TPC + j; byte offsets of their rows' windows in a B/C box
    constexpr int NWIN = TB / WT;
    constexpr bool OFF_TABLE = S * NWIN <= 16;
    int boff[OFF_TABLE ? S * NWIN : S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        if constexpr (OFF_TABLE) {
#pragma unroll
            for (int w = 0; w < NWIN; ++w) boff[s * NWIN + w] = bc_off<ESZ, TB>(s * TPC + j, w * WT);
        } else {
            boff[s] = s * TPC + j;
        }
    }

    float a2[NA], h[S];
    float Dd = 0.f, bias = 0.f;
#pragma unroll
    for (int s = 0; s < NA; ++s) a2[s] = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) h[s] = 0.f;

    for (unsigned c = 0;; ++c) {
        const int st = c % NST;
        unsigned char* sb = smem + Cf::OFF_STAGES + st * Cf::STAGE;
        if (!__all_sync(0xffffffffu, mbar_wait(bars + BAR_FULL + st, (c / NST) & 1, budget, status))) break;
        const BlockHdr hd = *reinterpret_cast<const BlockHdr*>(sb + Cf::OFF_HDR);
        if (hd.flags & kEnd) break;
        const int64_t ci = hd.ci0 + lc;
        const bool ok = ci < Dg;
        const int64_t d = hd.g * Dg + (ok ? ci : 0);
        const int64_t t0 = hd.t0;
        if (hd.flags & kFirst) {
            const float* ps = reinterpret_cast<const float*>(smem + Cf::OFF_PSLOT) + hd.pslot * Cf::PSLOT;
            const int64_t h_lo = (hd.g * Dg + hd.ci0) / P;
            const int hrel = ok ? (int)(d / P - h_lo) : 0;
            if constexpr (HEAD_A) {
                a2[0] = ps[Cf::P_A + hd.oa + hrel] * kLog2e;
            } else {
#pragma unroll
                for (int s = 0; s < S; ++s) a2[s] = ps[Cf::P_A + hd.oa + lc * N + s * TPC + j] * kLog2e;
            }
            Dd = ps[Cf::P_D + hd.od + lc];
            bias = ps[Cf::P_BIAS + hd.ob + hrel];
#pragma unroll
            for (int s = 0; s < S; ++s) h[s] = ps[Cf::P_H + lc * N + s * TPC + j];
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + BAR_PEMPTY + hd.pslot);
        }
        const unsigned char* urow = sb + Cf::OFF_IN + lc * RB + j * TPT * ESZ;
        const int64_t drow_i = HEAD_A ? (d / P - (hd.g * Dg + hd.ci0) / P) : lc;
        const unsigned char* drow = sb + Cf::OFF_IN + (CT + drow_i) * RB + j * TPT * ESZ;
        const unsigned char* zrow = sb + Cf::OFF_IN + (2 * CT + lc) * RB + j * TPT * ESZ;
        const bool full_blk = t0 + TB <= hd.t1;
        // the backward's stored states (CKPT): this lane's first state entering each 8-step
        // window of the block, and whether the lane's row is in bounds
        static_assert(Cf::WT == 4 || Cf::WT == 8, "windows on 8-step bounds");
        float* ckp = nullptr;
        bool ck0 = false;
        if constexpr (CKPT) {
            ckp = p.ckpt + ((hd.b * Dm + d) * p.ckpt_wins + t0 / 8) * N + j;
            ck0 = ok && in_bounds(hd.b < p.batch && d < Dm && t0 < L, status);
        }
        // -------- prologue: dt, dt*u (dA) of this lane's steps, two at a time
        {
            Chunk<T, TPT> cu, cd;
#pragma unroll
            for (int q = 0; q < Chunk<T, TPT>::kWords; ++q) {
                cu.w[q] = reinterpret_cast<const uint32_t*>(urow)[q];
                cd.w[q] = reinterpret_cast<const uint32_t*>(drow)[q];
            }
            float vdt[TPT], vdu[TPT];
#pragma unroll
            for (int i = 0; i < TPT; i += 2) {
                const float2 x = add2(IO<T>::get2(cd.w, i), dup2(bias));
                float2 dt = p.softplus ? softplus2(x) : x;
                if (!full_blk) {
                    // steps past the end of the unit: no step (dA = 1, no input); their u is zero-filled
                    if (t0 + j * TPT + i >= hd.t1) dt.x = 0.f;
                    if (t0 + j * TPT + i + 1 >= hd.t1) dt.y = 0.f;
                }
                const float2 du = mul2(dt, IO<T>::get2(cu.w, i));
                vdt[i] = dt.x; vdt[i + 1] = dt.y;
                vdu[i] = du.x; vdu[i + 1] = du.y;
            }
#pragma unroll
            for (int i = 0; i < TPT; i += 4) {
                *reinterpret_cast<float4*>(rdt + j * TPT + i) = make_float4(vdt[i], vdt[i + 1], vdt[i + 2], vdt[i + 3]);
                *reinterpret_cast<float4*>(rdu + j * TPT + i) = make_float4(vdu[i], vdu[i + 1], vdu[i + 2], vdu[i + 3]);
            }
            if constexpr (HEAD_A) {
#pragma unroll
                for (int i = 0; i < TPT; i += 4)
                    *reinterpret_cast<float4*>(rda + j * TPT + i) =
                        make_float4(ex2_approx(vdt[i] * a2[0]), ex2_approx(vdt[i + 1] * a2[0]),
                                    ex2_approx(vdt[i + 2] * a2[0]), ex2_approx(vdt[i + 3] * a2[0]));
            }
        }
        __syncwarp();
        // -------- the recurrence, one window of WT steps at a time (unrolled)
        const unsigned char* bcb = sb + Cf::OFF_BC;
        // A window's B and C words and its dt, dt*u (dA) rows, into register set bsel.  With
        // per-lane y rows (up to 8 consumer warps, registers to spare) the next window's set
        // is loaded while the current one runs (up to 4 states per lane); otherwise each
        // window loads its own.
        constexpr bool PF = Cf::YLANE && S <= 4;
        uint32_t bwA[PF ? 2 : 1][S][WT * ESZ / 4], cwA[PF ? 2 : 1][S][WT * ESZ / 4];
        float dtA[PF ? 2 : 1][WT], duA[PF ? 2 : 1][WT], daA[PF ? 2 : 1][HEAD_A ? WT : 1];
        auto load_window = [&](const int w, const int bsel) {
            const int tw = w * WT;
#pragma unroll
            for (int s = 0; s < S; ++s) {
                int off;
                if constexpr (OFF_TABLE) off = boff[s * NWIN + w];
                else off = bc_off<ESZ, TB>(boff[s], tw);
                const unsigned char* rb = bcb + off;
                const unsigned char* rc = bcb + N * RB + off;
                if constexpr (WT * ESZ == 16) {
                    const uint4 vb = *reinterpret_cast<const uint4*>(rb);
                    const uint4 vc = *reinterpret_cast<const uint4*>(rc);
                    bwA[bsel][s][0] = vb.x; bwA[bsel][s][1] = vb.y; bwA[bsel][s][2] = vb.z; bwA[bsel][s][3] = vb.w;
                    cwA[bsel][s][0] = vc.x; cwA[bsel][s][1] = vc.y; cwA[bsel][s][2] = vc.z; cwA[bsel][s][3] = vc.w;
                } else {
                    const uint2 vb = *reinterpret_cast<const uint2*>(rb);
                    const uint2 vc = *reinterpret_cast<const uint2*>(rc);
                    bwA[bsel][s][0] = vb.x; bwA[bsel][s][1] = vb.y;
                    cwA[bsel][s][0] = vc.x; cwA[bsel][s][1] = vc.y;
                }
            }
#pragma unroll
            for (int q = 0; q < WT; q += 4) {
                const float4 a4 = *reinterpret_cast<const float4*>(rdt + tw + q);
                const float4 bq = *reinterpret_cast<const float4*>(rdu + tw + q);
                dtA[bsel][q] = a4.x; dtA[bsel][q + 1] = a4.y; dtA[bsel][q + 2] = a4.z; dtA[bsel][q + 3] = a4.w;
                duA[bsel][q] = bq.x; duA[bsel][q + 1] = bq.y; duA[bsel][q + 2] = bq.z; duA[bsel][q + 3] = bq.w;
                if constexpr (HEAD_A) {
                    const float4 cq = *reinterpret_cast<const float4*>(rda + tw + q);
                    daA[bsel][q] = cq.x; daA[bsel][q + 1] = cq.y; daA[bsel][q + 2] = cq.z; daA[bsel][q + 3] = cq.w;
                }
            }
        };
        if constexpr (PF) load_window(0, 0);
#pragma unroll
        for (int w = 0; w < NWIN; ++w) {
            const int tw = w * WT;
            const int bsel = PF ? (w & 1) : 0;
            if constexpr (PF) {
                if (w + 1 < NWIN) load_window(w + 1, (w + 1) & 1);
            } else {
                load_window(w, 0);
            }
            // the state entering an 8-step window, for the backward (blocks start on 8-step
            // bounds).  Predicated stores, not a branch: the unrolled windows stay one stretch
            // of straight-line code for the scheduler.
            if (CKPT && (tw & 7) == 0) {
                const bool ckw = tw == 0 ? ck0 : ck0 && t0 + tw < hd.t1;
#pragma unroll
                for (int s = 0; s < S; ++s) st_global_if(ckp + (tw / 8) * N + s * TPC, h[s], ckw);
            }
            const auto& bw = bwA[bsel];
            const auto& cw_ = cwA[bsel];
            const auto& dtv = dtA[bsel];
            const auto& duv = duA[bsel];
            const auto& dav = daA[bsel];
            (void)dav;
            float yw[WT];
#pragma unroll
            for (int tt = 0; tt < WT; ++tt) {
                const float2 dt2 = dup2(dtv[tt]);
                const float2 du2 = dup2(duv[tt]);
                float2 y2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int s = 0; s < S; s += 2) {
                    float2 dA;
                    if constexpr (HEAD_A) {
                        dA = dup2(dav[tt]);
                    } else {
                        const float2 arg = mul2(dt2, make_float2(a2[s], a2[s + 1]));
                        dA = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                    }
                    const float2 bb = make_float2(IO<T>::get(bw[s], tt), IO<T>::get(bw[s + 1], tt));
                    const float2 cc = make_float2(IO<T>::get(cw_[s], tt), IO<T>::get(cw_[s + 1], tt));
                    const float2 hh = fma2(dA, make_float2(h[s], h[s + 1]), mul2(du2, bb));
                    h[s] = hh.x;
                    h[s + 1] = hh.y;
                    y2 = fma2(cc, hh, y2);
                }
                yw[tt] = y2.x + y2.y;
            }
            if constexpr (Cf::YLANE) {
                // this lane's partial sums to its own row (the window lies in the columns of one lane)
                float* yl = ry + j * Cf::YROW + tw + 4 * Cf::ysh(tw / TPT);
                *reinterpret_cast<float4*>(yl) = make_float4(yw[0], yw[1], yw[2], yw[3]);
                *reinterpret_cast<float4*>(yl + 4) = make_float4(yw[4], yw[5], yw[6], yw[7]);
            } else if constexpr (Cf::YPART) {
                // the first reduction round: the lower-half lane keeps steps 0-3 of the window
                const bool up = (j & 4) != 0;
                float rv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) rv[i] = __shfl_xor_sync(0xffffffffu, up ? yw[i] : yw[4 + i], 4);
                const float2 s0 = add2(up ? make_float2(yw[4], yw[5]) : make_float2(yw[0], yw[1]), make_float2(rv[0], rv[1]));
                const float2 s1 = add2(up ? make_float2(yw[6], yw[7]) : make_float2(yw[2], yw[3]), make_float2(rv[2], rv[3]));
                *reinterpret_cast<float4*>(ry + (j & 3) * Cf::YPROW + (up ? Cf::YHALF : 0) + tw / 2) =
                    make_float4(s0.x, s0.y, s1.x, s1.y);
            } else {
                int off;
                window_reduce<WT, TPC>(yw, j, off);
                if (j % (TPC > WT ? TPC / WT : 1) == 0) {
#pragma unroll
                    for (int i = 0; i < (WT >= TPC ? WT / TPC : 1); ++i) ry[tw + off + i] = yw[i];
                }
            }
        }
        // -------- end of a unit: the state goes to the outgoing slot (or last_state)
        if (hd.flags & kLast) {
            if (!(hd.flags & kFinalSeg)) {
                const int slot = hd.cseq & 1;
                if (hd.cseq >= 2)
                    __all_sync(0xffffffffu, mbar_wait(bars + BAR_CEMPTY + slot, ((hd.cseq >> 1) - 1) & 1, budget, status));
                float* cs = reinterpret_cast<float*>(smem + Cf::OFF_CSLOT) + slot * Cf::CSLOT;
#pragma unroll
                for (int s = 0; s < S; ++s) cs[lc * N + s * TPC + j] = h[s];
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + BAR_CFULL + slot);
            } else if (ok && p.last_state && in_bounds(hd.b < p.batch && d < Dm, status)) {
#pragma unroll
                for (int s = 0; s < S; ++s) p.last_state[((int64_t)hd.b * Dm + d) * N + s * TPC + j] = h[s];
            }
        }
        __syncwarp();
        // -------- epilogue: (y + D u) * silu(z) for the lane's own steps, two at a time
        {
            Chunk<T, TPT> cu, cz;
#pragma unroll
            for (int q = 0; q < Chunk<T, TPT>::kWords; ++q) {
                cu.w[q] = reinterpret_cast<const uint32_t*>(urow)[q];
                cz.w[q] = reinterpret_cast<const uint32_t*>(zrow)[q];
            }
            float o[TPT];
            if constexpr (Cf::YLANE) {
                // y of this lane's steps: the sum of the channel's TPC rows, added in the tree
                // the shuffle reduction uses (rows r and r + m for m = TPC/2, ..., 1), so both
                // readouts round alike
                const float* yc = ry + j * TPT + 4 * Cf::ysh(j);
#pragma unroll
                for (int i = 0; i < TPT; i += 4) {
                    float2 lo[TPC], hi[TPC];
#pragma unroll
                    for (int r = 0; r < TPC; ++r) {
                        const float4 w4 = *reinterpret_cast<const float4*>(yc + r * Cf::YROW + i);
                        lo[r] = make_float2(w4.x, w4.y);
                        hi[r] = make_float2(w4.z, w4.w);
                    }
#pragma unroll
                    for (int m = TPC / 2; m >= 1; m >>= 1) {
#pragma unroll
                        for (int r = 0; r < m; ++r) {
                            lo[r] = add2(lo[r], lo[r + m]);
                            hi[r] = add2(hi[r], hi[r + m]);
                        }
                    }
                    o[i] = lo[0].x; o[i + 1] = lo[0].y; o[i + 2] = hi[0].x; o[i + 3] = hi[0].y;
                }
            } else if constexpr (Cf::YPART) {
                // this lane's steps are window j: the 4 rows' halves, added in the shuffle tree's order
                float4 lo[4], hi[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    lo[r] = *reinterpret_cast<const float4*>(ry + r * Cf::YPROW + 4 * j);
                    hi[r] = *reinterpret_cast<const float4*>(ry + r * Cf::YPROW + Cf::YHALF + 4 * j);
                }
#pragma unroll
                for (int m = 2; m >= 1; m >>= 1) {
#pragma unroll
                    for (int r = 0; r < m; ++r) {
                        const float2 a = add2(make_float2(lo[r].x, lo[r].y), make_float2(lo[r + m].x, lo[r + m].y));
                        const float2 b = add2(make_float2(lo[r].z, lo[r].w), make_float2(lo[r + m].z, lo[r + m].w));
                        const float2 c = add2(make_float2(hi[r].x, hi[r].y), make_float2(hi[r + m].x, hi[r + m].y));
                        const float2 e = add2(make_float2(hi[r].z, hi[r].w), make_float2(hi[r + m].z, hi[r + m].w));
                        lo[r] = make_float4(a.x, a.y, b.x, b.y);
                        hi[r] = make_float4(c.x, c.y, e.x, e.y);
                    }
                }
                o[0] = lo[0].x; o[1] = lo[0].y; o[2] = lo[0].z; o[3] = lo[0].w;
                o[4] = hi[0].x; o[5] = hi[0].y; o[6] = hi[0].z; o[7] = hi[0].w;
            } else {
#pragma unroll
                for (int i = 0; i < TPT; i += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(ry + j * TPT + i);
                    o[i] = v.x; o[i + 1] = v.y; o[i + 2] = v.z; o[i + 3] = v.w;
                }
            }
#pragma unroll
            for (int i = 0; i < TPT; i += 2) {
                float2 v = fma2(dup2(Dd), IO<T>::get2(cu.w, i), make_float2(o[i], o[i + 1]));
                if (p.z) v = mul2(v, silu2(IO<T>::get2(cz.w, i)));
                o[i] = v.x;
                o[i + 1] = v.y;
            }
            const int64_t tl = t0 + j * TPT;
            if (ok && tl < hd.t1 && in_bounds(hd.b < p.batch && d < Dm && tl >= 0 && hd.t1 <= L, status)) {
                T* orow = reinterpret_cast<T*>(p.out) + (hd.b * Dm + d) * L;
                store_chunk<T, TPT, VEC>(orow, tl, hd.t1, o);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + BAR_EMPTY + st);
    }
}

// ------------------------------------------------------- tensor-memory kernel
//
// The same scan for bf16 I/O with 16 states, with B and C brought to the
// consumers through tensor memory instead of shared memory.  Per 32-step block, a
// tensor-core warp issues one-hot MMAs (kind::f16, M = 128 TMEM lanes, N = TS
// steps, K = 16 states): TMEM lane i (consumer lane i % 32 of its warp) receives,
// for each of its S state slots s, B[n][t] and C[n][t] of state n = s*TPC + j for
// the TS steps of its time sub-chunk k, as fp32 (KT = 1: one sub-chunk of all 32
// steps).  The sub-chunk is folded into the product: slice (s, k) of the one-hot
// operand selects the lanes of sub-chunk k, and its MMA reads the B or C box from
// step k*TS on, accumulating into the same columns, so every lane of a warp finds
// its own steps at the same TMEM columns.  A one-hot product adds one bf16 value
// times 1.0 to zeros, so the copy is exact.
// The consumers read their columns with tcgen05.ld, so B and C cost no shared-memory
// bandwidth and no bf16 unpacking.  The recurrence pairs two consecutive steps of a
// state in the f32x2 operations (dt, dt*u, B and C of steps t, t+1 are adjacent in
// their rows and columns), with the state update itself two scalar FMAs.  The
// lanes' partial sums of y go to per-lane rows in shared memory; the epilogue adds
// the TPC rows of each step.

template <int W, int SPL, int KT>
struct CfgTc {
    using Elem = __nv_bfloat16;
    static constexpr bool kHeadA = false;
    static constexpr int kN = 16;
    static constexpr int N = 16;
    static constexpr int ESZ = 2;
    static constexpr int S = SPL;                          // states per lane
    static constexpr int TPC = N / S;                      // lanes per channel and time sub-chunk
    static constexpr int TPCS = TPC * KT;                  // lanes per channel
    static constexpr int TS = kTB / KT;                    // steps of a time sub-chunk
    static constexpr int GW = 32 / TPCS;                   // channels per consumer warp
    static constexpr int CT = W * GW;                      // channels per tile
    static constexpr int TPT = kTB / TPCS;                 // steps per lane in prologue / epilogue
    static constexpr int RB = kTB * ESZ;                   // bytes of one block row
    static constexpr int WIN = KT == 1 ? 8 : 4;            // steps per tensor-memory read
    static constexpr int TB = kTB;                         // steps per block
    static constexpr int NSLICE = S * KT;                  // one-hot K-slices (16 columns each)
    // one ring stage (1024-byte aligned): B box | C box (16 rows of 64 bytes each, 64-byte
    // swizzle, read by the tensor cores as an MN-major operand) | u box | delta box | z box
    // (CT rows each) | header
    static constexpr int OFF_BC = 0;
    static constexpr int OFF_IN = OFF_BC + 2 * N * RB;
    static constexpr int OFF_HDR = OFF_IN + 3 * CT * RB;
    static constexpr int STAGE = (OFF_HDR + 64 + 1023) / 1024 * 1024;
    // unit parameter slot (floats), outgoing state slot (floats), as in Cfg
    static constexpr int P_A = 0;
    static constexpr int P_D = P_A + CT * N + 8;
    static constexpr int P_BIAS = P_D + CT + 8;
    static constexpr int P_H = P_BIAS + CT + 8;
    static constexpr int PSLOT = P_H + CT * N;
    static constexpr int CSLOT = CT * N;
    // per consumer warp (floats): dt and dt*u rows per channel, then one row of partial
    // sums of y per lane
    static constexpr int ROW = kTB + 4;                    // 144 bytes: rows start in different banks
    static constexpr int W_DT = 0;
    static constexpr int W_DU = GW * ROW;
    static constexpr int W_Y = 2 * GW * ROW;
    static constexpr int WARP_F = W_Y + 32 * ROW;
    // tensor memory: per block, S groups of TS columns for B then S for C; NB blocks in flight
    static constexpr int TC_BLK = 2 * S * TS;
    static constexpr int NB = 512 / TC_BLK > 4 ? 4 : 512 / TC_BLK;
    // shared memory map (bytes): barriers | stages | one-hot operand (128 rows x 128 bytes,
    // K-major, 128-byte swizzle) | parameter slots | outgoing slots | per-warp rows
    static constexpr int OFF_STAGES = 1024;
    static constexpr int ONEHOT = 128 * 128;
    static constexpr int REST = ONEHOT + 2 * PSLOT * 4 + 2 * CSLOT * 4 + W * WARP_F * 4;
    static constexpr int STG = OFF_STAGES + kStages * STAGE + REST <= 227 * 1024 ? kStages : 2;
    static constexpr int OFF_ONEHOT = OFF_STAGES + STG * STAGE;
    static constexpr int OFF_PSLOT = OFF_ONEHOT + ONEHOT;
    static constexpr int OFF_CSLOT = OFF_PSLOT + 2 * PSLOT * 4;
    static constexpr int OFF_WARP = OFF_CSLOT + 2 * CSLOT * 4;
    static constexpr int SMEM = OFF_WARP + W * WARP_F * 4;
    static constexpr int THREADS = 32 * (W + 2);           // consumers, the producer, the tensor-core warp
    static constexpr bool kFits = SMEM <= 227 * 1024;
    static_assert(S % 2 == 0 && N % S == 0 && TPC >= 2 && TPC <= 8, "lane split");
    static_assert((KT == 1 || KT == 2) && TPCS <= 32 && TS % WIN == 0 && TS % 16 == 0, "time sub-chunks");
    static_assert(TPT % 2 == 0 && TPT <= 16, "steps per lane must be 2..16");
    static_assert(STAGE % 1024 == 0 && (PSLOT * 4) % 16 == 0 && (WARP_F * 4) % 16 == 0, "aligned smem");
    static_assert(NSLICE <= 4, "the one-hot slices fit one 128-byte row");
};

// barrier slots of the tensor-memory kernel (the TMEM base address sits at byte 512)
enum { BT_RAW = 0, BT_EMPTY = kStages, BT_TFULL = 2 * kStages, BT_TEMPTY = 2 * kStages + 4,
       BT_PEMPTY = 2 * kStages + 8, BT_CFULL = 2 * kStages + 10, BT_CEMPTY = 2 * kStages + 12,
       BT_DONE = 2 * kStages + 14 };
constexpr int kTmemAddrOff = 512;
static_assert((2 * kStages + 15) * 8 <= kTmemAddrOff, "barriers fit below the TMEM address");

// 8 consecutive 32-bit TMEM columns of this thread's lane (registers valid after tc::wait_ld)
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

// 4 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
template <int R>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[R]) {
    if constexpr (R == 8) tmem_ld8(taddr, r);
    else tmem_ld4(taddr, r);
}
// ties registers loaded from tensor memory to the preceding tcgen05.wait::ld
template <int R>
__device__ __forceinline__ void tmem_after_wait(uint32_t (&r)[R]) {
#pragma unroll
    for (int i = 0; i < R; i += 4) asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]));
}

template <int W, int SPL, int KT, bool VEC>
__global__ void __launch_bounds__(CfgTc<W, SPL, KT>::THREADS, 1)
scan_fwd_tc_kernel(const FwdParams p, const __grid_constant__ TensorMaps tm) {
    using Cf = CfgTc<W, SPL, KT>;
    using T = __nv_bfloat16;
    constexpr int N = Cf::N, S = Cf::S, TPC = Cf::TPC, TPCS = Cf::TPCS, TS = Cf::TS, GW = Cf::GW, CT = Cf::CT;
    constexpr int TPT = Cf::TPT, ESZ = Cf::ESZ, RB = Cf::RB, WIN = Cf::WIN, NB = Cf::NB, TC_BLK = Cf::TC_BLK;
    constexpr int NST = Cf::STG;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemAddrOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Dm = p.dim, L = p.seqlen, G = p.ngroups;
    const int64_t Dg = Dm / G;
    int* status = &p.ws->status;
    const uint64_t budget = (uint64_t)p.spin_limit * 256ull;  // ns

    // the swizzles of the boxes and of the one-hot operand assume a 1024-byte aligned base
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(status, SSM_OK, SSM_ERR_BOUNDS);
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bars + BT_RAW + s, 1);
            mbar_init(bars + BT_EMPTY + s, W);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(bars + BT_TFULL + b, 1);
            mbar_init(bars + BT_TEMPTY + b, W);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bars + BT_PEMPTY + s, W);
            mbar_init(bars + BT_CFULL + s, W);
            mbar_init(bars + BT_CEMPTY + s, 1);
        }
        mbar_init(bars + BT_DONE, W);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the one-hot operand: K-slice q = s*KT + kk (columns 16q .. 16q+15) of row i (a TMEM
    // lane, consumer lane l = i % 32 with state group l % TPC and sub-chunk (l % TPCS) / TPC)
    // has a 1 in the column of state n = s*TPC + l % TPC if the lane's sub-chunk is kk;
    // written in 16-byte pieces
    {
        unsigned char* oh = smem + Cf::OFF_ONEHOT;
        for (int e = threadIdx.x; e < 128 * 8; e += Cf::THREADS) {
            const int i = e >> 3, c8 = (e & 7) * 8, l = i & 31;
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int col = c8 + q, sl = col >> 4, s = sl / KT, kk = sl % KT;
                if (sl < Cf::NSLICE && (l % TPCS) / TPC == kk && (col & 15) == s * TPC + l % TPC)
                    w4[q >> 1] |= 0x3F80u << (16 * (q & 1));
            }
            *reinterpret_cast<uint4*>(oh + tc::sw128_off(i, c8)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        tc::fence_async_smem();
    }
    if (warp == W + 1) tc::alloc(tmem_slot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == W) {
        // ============================================================ producer
        produce<Cf, VEC>(p, tm, smem,
                         ProducerBars{bars + BT_RAW, bars + BT_EMPTY, bars + BT_PEMPTY, bars + BT_CFULL,
                                      bars + BT_CEMPTY},
                         lane, budget, status);
        return;
    }

    if (warp == W + 1) {
        // ============================================================ tensor cores
        // per block: wait for its copies and for a free TMEM buffer, then 2*S*KT one-hot MMAs
        constexpr uint32_t idesc = tc::idesc_bf16(128, TS, false, true);
        const uint64_t a0 = tc::desc(smem + Cf::OFF_ONEHOT, 16, 1024, tc::kSwizzle128);
        unsigned issued = 0;
        for (unsigned c = 0;; ++c) {
            const int st = c % NST, buf = c % NB;
            unsigned char* sb = smem + Cf::OFF_STAGES + st * Cf::STAGE;
            if (!lane0_says(lane == 0 ? mbar_wait(bars + BT_RAW + st, (c / NST) & 1, budget, status) : false)) break;
            __syncwarp();
            const int flags = reinterpret_cast<const BlockHdr*>(sb + Cf::OFF_HDR)->flags;
            if (flags & kEnd) break;
            if (c >= (unsigned)NB &&
                !lane0_says(lane == 0 ? mbar_wait(bars + BT_TEMPTY + buf, ((c / NB) - 1) & 1, budget, status) : false))
                break;
            tc::fence_after();
            if (lane == 0) {
                const uint32_t d0 = tbase + (uint32_t)(buf * TC_BLK);
#pragma unroll
                for (int kk = 0; kk < KT; ++kk) {
                    // the boxes from step kk*TS on (MN-major, 64-byte swizzle; one swizzle atom along
                    // the steps, so both strides are the 8-row step along the states)
                    const uint64_t bB = tc::desc(sb + Cf::OFF_BC + kk * TS * ESZ, 512, 512, tc::kSwizzle64);
                    const uint64_t bC = tc::desc(sb + Cf::OFF_BC + N * RB + kk * TS * ESZ, 512, 512, tc::kSwizzle64);
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        // K-slice s*KT + kk of the one-hot rows: +32 bytes per slice inside the swizzled row
                        const uint64_t a = a0 + (uint64_t)(((s * KT + kk) * 32) >> 4);
                        tc::mma_bf16(d0 + s * TS, a, bB, idesc, kk > 0 ? 1u : 0u);
                        tc::mma_bf16(d0 + (S + s) * TS, a, bC, idesc, kk > 0 ? 1u : 0u);
                    }
                }
                tc::commit(bars + BT_TFULL + buf);
            }
            __syncwarp();
            issued = c + 1;
        }
        // the last products have landed and every consumer warp is done with tensor memory
        // before it is freed (both waits bounded)
        if (issued > 0)
            lane0_says(lane == 0 ? mbar_wait(bars + BT_TFULL + (issued - 1) % NB, ((issued - 1) / NB) & 1, budget, status)
                                 : false);
        lane0_says(lane == 0 ? mbar_wait(bars + BT_DONE, 0, 4 * budget, status) : false);
        __syncwarp();
        tc::fence_after();
        tc::dealloc(tbase, 512);
        return;
    }

    // ================================================================ consumers
    // lane = (channel cg, time sub-chunk k, state group j): lane j of sub-chunk k holds
    // states n = s*TPC + j of channel cg for steps [k*TS, (k+1)*TS) of every block
    const int cg = lane / TPCS, jj = lane % TPCS;
    const int k = jj / TPC, j = jj % TPC;
    const int lc = warp * GW + cg;   // channel of the lane within the tile
    float* wf = reinterpret_cast<float*>(smem + Cf::OFF_WARP) + warp * Cf::WARP_F;
    float* rdt = wf + Cf::W_DT + cg * Cf::ROW;
    float* rdu = wf + Cf::W_DU + cg * Cf::ROW;
    float* yrow = wf + Cf::W_Y + lane * Cf::ROW;
    const float* ych = wf + Cf::W_Y + cg * TPCS * Cf::ROW;
    const uint32_t tlane = tbase + ((uint32_t)((warp & 3) * 32) << 16);

    float2 a2p[S];   // (A log2 e, A log2 e) per state
    float h[S];
    float Dd = 0.f, bias = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
        a2p[s] = make_float2(0.f, 0.f);
        h[s] = 0.f;
    }

    for (unsigned c = 0;; ++c) {
        const int st = c % NST, buf = c % NB;
        unsigned char* sb = smem + Cf::OFF_STAGES + st * Cf::STAGE;
        if (!__all_sync(0xffffffffu, mbar_wait(bars + BT_RAW + st, (c / NST) & 1, budget, status))) break;
        const BlockHdr hd = *reinterpret_cast<const BlockHdr*>(sb + Cf::OFF_HDR);
        if (hd.flags & kEnd) break;
        const int64_t ci = hd.ci0 + lc;
        const bool ok = ci < Dg;
        const int64_t d = hd.g * Dg + (ok ? ci : 0);
        const int64_t t0 = hd.t0;
        if (hd.flags & kFirst) {
            const float* ps = reinterpret_cast<const float*>(smem + Cf::OFF_PSLOT) + hd.pslot * Cf::PSLOT;
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const float a = ps[Cf::P_A + hd.oa + lc * N + s * TPC + j] * kLog2e;
                a2p[s] = make_float2(a, a);
                h[s] = ps[Cf::P_H + lc * N + s * TPC + j];
            }
            Dd = ps[Cf::P_D + hd.od + lc];
            bias = ps[Cf::P_BIAS + hd.ob + lc];
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + BT_PEMPTY + hd.pslot);
        }
        const unsigned char* urow = sb + Cf::OFF_IN + lc * RB + jj * TPT * ESZ;
        const unsigned char* drow = sb + Cf::OFF_IN + (CT + lc) * RB + jj * TPT * ESZ;
        const unsigned char* zrow = sb + Cf::OFF_IN + (2 * CT + lc) * RB + jj * TPT * ESZ;
        const bool full_blk = t0 + kTB <= hd.t1;
        // -------- prologue: dt and dt*u of this lane's steps into the channel's rows
        {
            Chunk<T, TPT> cu, cd;
#pragma unroll
            for (int q = 0; q < Chunk<T, TPT>::kWords; ++q) {
                cu.w[q] = reinterpret_cast<const uint32_t*>(urow)[q];
                cd.w[q] = reinterpret_cast<const uint32_t*>(drow)[q];
            }
#pragma unroll
            for (int i = 0; i < TPT; i += 2) {
                const float2 x = add2(IO<T>::get2(cd.w, i), dup2(bias));
                float2 dt = p.softplus ? softplus2(x) : x;
                if (!full_blk) {
                    // steps past the end of the unit: no step (dA = 1, no input); their u is zero-filled
                    if (t0 + jj * TPT + i >= hd.t1) dt.x = 0.f;
                    if (t0 + jj * TPT + i + 1 >= hd.t1) dt.y = 0.f;
                }
                const float2 du = mul2(dt, IO<T>::get2(cu.w, i));
                *reinterpret_cast<float2*>(rdt + jj * TPT + i) = dt;
                *reinterpret_cast<float2*>(rdu + jj * TPT + i) = du;
            }
        }
        __syncwarp();
        // -------- B and C of the block in tensor memory
        if (!__all_sync(0xffffffffu, mbar_wait(bars + BT_TFULL + buf, (c / NB) & 1, budget, status))) break;
        tc::fence_after();
        // -------- the recurrence over the lane's steps, two steps of a state at a time
        {
            const int tb = k * TS;
            const uint32_t tcol = tlane + (uint32_t)(buf * TC_BLK);
            if constexpr (KT == 1) {
#pragma unroll 1
                for (int w0 = 0; w0 < kTB; w0 += WIN) {
                    uint32_t rb[S][WIN], rc[S][WIN];
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        tmem_ld(tcol + s * TS + w0, rb[s]);
                        tmem_ld(tcol + (S + s) * TS + w0, rc[s]);
                    }
                    tc::wait_ld();
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        tmem_after_wait(rb[s]);
                        tmem_after_wait(rc[s]);
                    }
                    float dtv[WIN], duv[WIN];
#pragma unroll
                    for (int q = 0; q < WIN; q += 4) {
                        const float4 a = *reinterpret_cast<const float4*>(rdt + w0 + q);
                        const float4 b = *reinterpret_cast<const float4*>(rdu + w0 + q);
                        dtv[q] = a.x; dtv[q + 1] = a.y; dtv[q + 2] = a.z; dtv[q + 3] = a.w;
                        duv[q] = b.x; duv[q + 1] = b.y; duv[q + 2] = b.z; duv[q + 3] = b.w;
                    }
                    float yv[WIN];
#pragma unroll
                    for (int q = 0; q < WIN; q += 2) {
                        const float2 dt2 = make_float2(dtv[q], dtv[q + 1]);
                        const float2 du2 = make_float2(duv[q], duv[q + 1]);
                        float2 y2;
#pragma unroll
                        for (int s = 0; s < S; ++s) {
                            const float2 arg = mul2(dt2, a2p[s]);
                            const float2 dA = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                            const float2 bu = mul2(du2, make_float2(__uint_as_float(rb[s][q]), __uint_as_float(rb[s][q + 1])));
                            const float h0 = fmaf(dA.x, h[s], bu.x);
                            h[s] = fmaf(dA.y, h0, bu.y);
                            const float2 cc = make_float2(__uint_as_float(rc[s][q]), __uint_as_float(rc[s][q + 1]));
                            y2 = s == 0 ? mul2(cc, make_float2(h0, h[s])) : fma2(cc, make_float2(h0, h[s]), y2);
                        }
                        yv[q] = y2.x;
                        yv[q + 1] = y2.y;
                    }
#pragma unroll
                    for (int q = 0; q < WIN; q += 4)
                        *reinterpret_cast<float4*>(yrow + w0 + q) = make_float4(yv[q], yv[q + 1], yv[q + 2], yv[q + 3]);
                }
            } else {
                // Sequence-parallel block: sub-chunk k runs its TS steps from h = 0 (sub-chunk 0
                // from the carried state) and keeps v_t = C_t * prod(dA) over the sub-chunk so
                // far; an inclusive scan of the sub-chunks' (prod dA, end state) pairs over the KT
                // lanes that share (channel, j), with (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2),
                // gives each sub-chunk its true start state h_start, and y_t += v_t . h_start
                // (h_t = h_local,t + prod(dA) h_start) fixes up the readout.
                float hl[S], pr[S];
                float yv[TS], vv[TS][S];
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    hl[s] = k == 0 ? h[s] : 0.f;
                    pr[s] = 1.f;
                }
#pragma unroll
                for (int w0 = 0; w0 < TS; w0 += WIN) {
                    uint32_t rb[S][WIN], rc[S][WIN];
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        tmem_ld(tcol + s * TS + w0, rb[s]);
                        tmem_ld(tcol + (S + s) * TS + w0, rc[s]);
                    }
                    tc::wait_ld();
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        tmem_after_wait(rb[s]);
                        tmem_after_wait(rc[s]);
                    }
#pragma unroll
                    for (int q = 0; q < WIN; q += 2) {
                        const float2 dt2 = *reinterpret_cast<const float2*>(rdt + tb + w0 + q);
                        const float2 du2 = *reinterpret_cast<const float2*>(rdu + tb + w0 + q);
                        float2 y2;
#pragma unroll
                        for (int s = 0; s < S; ++s) {
                            const float2 arg = mul2(dt2, a2p[s]);
                            const float2 dA = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                            const float2 bu = mul2(du2, make_float2(__uint_as_float(rb[s][q]), __uint_as_float(rb[s][q + 1])));
                            const float h0 = fmaf(dA.x, hl[s], bu.x);
                            hl[s] = fmaf(dA.y, h0, bu.y);
                            const float p0 = pr[s] * dA.x;
                            pr[s] = p0 * dA.y;
                            const float2 cc = make_float2(__uint_as_float(rc[s][q]), __uint_as_float(rc[s][q + 1]));
                            const float2 vc = mul2(cc, make_float2(p0, pr[s]));
                            vv[w0 + q][s] = vc.x;
                            vv[w0 + q + 1][s] = vc.y;
                            y2 = s == 0 ? mul2(cc, make_float2(h0, hl[s])) : fma2(cc, make_float2(h0, hl[s]), y2);
                        }
                        yv[w0 + q] = y2.x;
                        yv[w0 + q + 1] = y2.y;
                    }
                }
#pragma unroll
                for (int r = 1; r < KT; r <<= 1) {
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        const float pu = __shfl_up_sync(0xffffffffu, pr[s], TPC * r);
                        const float hu = __shfl_up_sync(0xffffffffu, hl[s], TPC * r);
                        if (k >= r) {
                            hl[s] = fmaf(pr[s], hu, hl[s]);
                            pr[s] *= pu;
                        }
                    }
                }
                float2 hs[S];
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const float up = __shfl_up_sync(0xffffffffu, hl[s], TPC);
                    hs[s] = k == 0 ? make_float2(0.f, 0.f) : make_float2(up, up);
                    h[s] = __shfl_sync(0xffffffffu, hl[s], cg * TPCS + (KT - 1) * TPC + j);
                }
#pragma unroll
                for (int q = 0; q < TS; q += 4) {
                    float2 y01 = make_float2(yv[q], yv[q + 1]), y23 = make_float2(yv[q + 2], yv[q + 3]);
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        y01 = fma2(make_float2(vv[q][s], vv[q + 1][s]), hs[s], y01);
                        y23 = fma2(make_float2(vv[q + 2][s], vv[q + 3][s]), hs[s], y23);
                    }
                    *reinterpret_cast<float4*>(yrow + tb + q) = make_float4(y01.x, y01.y, y23.x, y23.y);
                }
            }
        }
        // tensor memory of this block read: the tensor-core warp may refill the buffer
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + BT_TEMPTY + buf);
        // -------- end of a unit: the state goes to the outgoing slot (or last_state)
        if (hd.flags & kLast) {
            if (!(hd.flags & kFinalSeg)) {
                const int slot = hd.cseq & 1;
                if (hd.cseq >= 2)
                    __all_sync(0xffffffffu, mbar_wait(bars + BT_CEMPTY + slot, ((hd.cseq >> 1) - 1) & 1, budget, status));
                float* cs = reinterpret_cast<float*>(smem + Cf::OFF_CSLOT) + slot * Cf::CSLOT;
                if (k == 0) {
#pragma unroll
                    for (int s = 0; s < S; ++s) cs[lc * N + s * TPC + j] = h[s];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + BT_CFULL + slot);
            } else if (ok && p.last_state && k == 0 && in_bounds(hd.b < p.batch && d < Dm, status)) {
#pragma unroll
                for (int s = 0; s < S; ++s) p.last_state[((int64_t)hd.b * Dm + d) * N + s * TPC + j] = h[s];
            }
        }
        __syncwarp();
        // -------- epilogue: y summed over the TPC lanes that hold the step's states, then
        // (y + D u) * silu(z) for the lane's own steps, two at a time
        {
            Chunk<T, TPT> cu, cz;
#pragma unroll
            for (int q = 0; q < Chunk<T, TPT>::kWords; ++q) {
                cu.w[q] = reinterpret_cast<const uint32_t*>(urow)[q];
                cz.w[q] = reinterpret_cast<const uint32_t*>(zrow)[q];
            }
            const int t_l = jj * TPT;
            const float* yr = ych + (t_l / TS) * TPC * Cf::ROW + t_l;
            float o[TPT];
            if constexpr (TPT % 4 == 0) {
#pragma unroll
                for (int i = 0; i < TPT; i += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(yr + i);
                    float2 lo = make_float2(v.x, v.y), hi = make_float2(v.z, v.w);
#pragma unroll
                    for (int r = 1; r < TPC; ++r) {
                        const float4 q = *reinterpret_cast<const float4*>(yr + r * Cf::ROW + i);
                        lo = add2(lo, make_float2(q.x, q.y));
                        hi = add2(hi, make_float2(q.z, q.w));
                    }
                    o[i] = lo.x; o[i + 1] = lo.y; o[i + 2] = hi.x; o[i + 3] = hi.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < TPT; i += 2) {
                    float2 acc = *reinterpret_cast<const float2*>(yr + i);
#pragma unroll
                    for (int r = 1; r < TPC; ++r) acc = add2(acc, *reinterpret_cast<const float2*>(yr + r * Cf::ROW + i));
                    o[i] = acc.x;
                    o[i + 1] = acc.y;
                }
            }
#pragma unroll
            for (int i = 0; i < TPT; i += 2) {
                float2 v = fma2(dup2(Dd), IO<T>::get2(cu.w, i), make_float2(o[i], o[i + 1]));
                if (p.z) v = mul2(v, silu2(IO<T>::get2(cz.w, i)));
                o[i] = v.x;
                o[i + 1] = v.y;
            }
            const int64_t tl = t0 + t_l;
            if (ok && tl < hd.t1 && in_bounds(hd.b < p.batch && d < Dm && tl >= 0 && hd.t1 <= L, status)) {
                T* orow = reinterpret_cast<T*>(p.out) + (hd.b * Dm + d) * L;
                store_chunk<T, TPT, VEC>(orow, tl, hd.t1, o);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + BT_EMPTY + st);
    }
    // this warp reads no more tensor memory
    tc::fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + BT_DONE);
}

// ------------------------------------------------------- segment policy

// Default segment length (steps, a multiple of every block length) for a launch of `ctas`
// persistent CTAs over `n_tiles` channel tiles of a sequence of L steps.
// Segments of one tile run one after another (each starts from the state the
// previous one published), so a segment is the unit of load balance: about
// eight per CTA keep the SMs evenly busy to the end, while every unit also pays
// a fixed start-up (parameter load, carry hand-off).  Measured on B200: short
// segments (64 steps) lose about a third of the throughput, and beyond eight
// units per CTA the gain flattens, so segments stay within [256, 2048] steps.
inline int64_t default_seg_len(int64_t L, int64_t n_tiles, int64_t ctas) {
    if (L <= 0) return kSegAlign;
    const int64_t t = n_tiles > 0 ? n_tiles : 1;
    int64_t n_seg = (8 * ctas + t - 1) / t;
    if (n_seg < 1) n_seg = 1;
    int64_t seg = (L + n_seg - 1) / n_seg;
    if (seg > 2048) seg = 2048;
    if (seg < 256) seg = 256;
    seg = (seg + kSegAlign - 1) / kSegAlign * kSegAlign;
    return seg;
}

// --------------------------------------------------------------- dispatch

using KernelFn = void (*)(const FwdParams, const TensorMaps);

struct Variant {
    KernelFn fn;
    int smem;
    int threads;
    int ch_per_tile;   // CT
    int dstate;
    int tb;            // steps per block (the tensor maps' box width)
    const char* name;
};

template <typename T, int N, int W, bool HEAD_A, int SPL, bool VEC, bool CKPT = false>
Variant make_variant(const char* name) {
    using C = Cfg<T, N, W, HEAD_A, SPL>;
    return Variant{scan_fwd_kernel<T, N, W, HEAD_A, SPL, VEC, CKPT>, C::SMEM, C::THREADS, C::CT, N, C::TB, name};
}
template <int W, int SPL, int KT, bool VEC>
Variant make_variant_tc(const char* name) {
    using C = CfgTc<W, SPL, KT>;
    return Variant{scan_fwd_tc_kernel<W, SPL, KT, VEC>, C::SMEM, C::THREADS, C::CT, 16, C::TB, name};
}

// The lane layouts compiled for a state size N: (consumer warps W, states per lane S).
// The register kernel (mode 0, KT = 1):
//   N <= 16: (16, 2), (8, 4), (8, 2), (4, 4), (4, 2), and (12, 4) for N = 16;
//   N = 32: (8, 4), (4, 4);
//   N >= 64: (8, N/8), (4, N/8).
// Mode 2 is the register kernel that also stores the states for the backward (N = 16, A
// per channel).
// The tensor-memory kernel (mode 1: bf16, N = 16, A per channel), with KT time sub-chunks
// per block: (16, 2, 1), (8, 4, 1), (12, 4, 1), (16, 2, 2), (8, 2, 2).
constexpr bool layout_listed(int N, int w, int spl) {
    if (N <= 16)
        return (w == 16 && spl == 2) || (N == 16 && w == 12 && spl == 4) ||
               ((w == 8 || w == 4) && (spl == 2 || spl == 4));
    if (N == 32) return (w == 8 || w == 4) && spl == 4;
    return (w == 8 || w == 4) && spl == N / 8;
}
// a listed layout whose lane split, steps per lane and shared-memory map work out
template <typename T, int N, int W, int SPL>
constexpr bool layout_exists() {
    if constexpr (layout_listed(N, W, SPL)) return Cfg<T, N, W, false, SPL>::kFits && Cfg<T, N, W, true, SPL>::kFits;
    else return false;
}
constexpr bool layout_exists_tc(int w, int spl, int kt) {
    return (kt == 1 && ((w == 16 && spl == 2) || ((w == 8 || w == 12) && spl == 4))) ||
           (kt == 2 && (w == 16 || w == 8) && spl == 2);
}
template <int W, int SPL, int KT>
constexpr bool tc_fits() {
    if constexpr (layout_exists_tc(W, SPL, KT)) return CfgTc<W, SPL, KT>::kFits;
    else return false;
}

// One function per (io dtype, N) translation unit; see fwd_*.cu.
#define SSM_PICK_ONE(T, TN, N, W, SPL)                                                                   \
    if ((mode == 0 || mode == 2) && kt == 1 && w == W && spl == SPL) {                                   \
        if constexpr (layout_exists<T, N, W, SPL>()) {                                                   \
            if (mode == 2) {                                                                             \
                if constexpr (N == 16) {                                                                 \
                    if (head) return false;                                                              \
                    *v = vec ? make_variant<T, N, W, false, SPL, true, true>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1_ckpt_vec") \
                             : make_variant<T, N, W, false, SPL, false, true>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1_ckpt"); \
                    return true;                                                                         \
                }                                                                                        \
                return false;                                                                            \
            }                                                                                            \
            if (head)                                                                                    \
                *v = vec ? make_variant<T, N, W, true, SPL, true>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1_head_vec") \
                         : make_variant<T, N, W, true, SPL, false>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1_head");   \
            else                                                                                         \
                *v = vec ? make_variant<T, N, W, false, SPL, true>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1_vec")     \
                         : make_variant<T, N, W, false, SPL, false>("ws_" #TN "_n" #N "_w" #W "s" #SPL "t1");          \
            return true;                                                                                 \
        }                                                                                                \
        return false;                                                                                    \
    }
#define SSM_PICK_TC(W, SPL, KT)                                                                          \
    if (mode == 1 && w == W && spl == SPL && kt == KT) {                                                 \
        if constexpr (tc_fits<W, SPL, KT>()) {                                                           \
            *v = vec ? make_variant_tc<W, SPL, KT, true>("tc_bf16_n16_w" #W "s" #SPL "t" #KT "_vec")       \
                     : make_variant_tc<W, SPL, KT, false>("tc_bf16_n16_w" #W "s" #SPL "t" #KT);            \
            return true;                                                                                 \
        }                                                                                                \
        return false;                                                                                    \
    }
#define SSM_DEFINE_PICK(T, TN, N)                                                                         \
    bool pick_##TN##_n##N(bool head, bool vec, int w, int spl, int kt, int mode, Variant* v) {           \
        SSM_PICK_ONE(T, TN, N, 16, 2)                                                                    \
        SSM_PICK_ONE(T, TN, N, 12, 4)                                                                    \
        SSM_PICK_ONE(T, TN, N, 8, 2)                                                                     \
        SSM_PICK_ONE(T, TN, N, 8, 4)                                                                     \
        SSM_PICK_ONE(T, TN, N, 4, 2)                                                                     \
        SSM_PICK_ONE(T, TN, N, 4, 4)                                                                     \
        SSM_PICK_ONE(T, TN, N, 8, 8)                                                                     \
        SSM_PICK_ONE(T, TN, N, 4, 8)                                                                     \
        SSM_PICK_ONE(T, TN, N, 8, 16)                                                                    \
        SSM_PICK_ONE(T, TN, N, 4, 16)                                                                    \
        return false;                                                                                    \
    }
// the tensor-memory variants (bf16, N = 16, A per channel)
#define SSM_DEFINE_PICK_TC                                                                                \
    bool pick_tc(bool vec, int w, int spl, int kt, int mode, Variant* v) {                                \
        SSM_PICK_TC(16, 2, 1)                                                                            \
        SSM_PICK_TC(8, 4, 1)                                                                             \
        SSM_PICK_TC(12, 4, 1)                                                                            \
        SSM_PICK_TC(16, 2, 2)                                                                            \
        SSM_PICK_TC(8, 2, 2)                                                                             \
        return false;                                                                                    \
    }

#define SSM_DECLARE_PICK(TN, N) bool pick_##TN##_n##N(bool head, bool vec, int w, int spl, int kt, int mode, Variant* v);
bool pick_tc(bool vec, int w, int spl, int kt, int mode, Variant* v);
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
