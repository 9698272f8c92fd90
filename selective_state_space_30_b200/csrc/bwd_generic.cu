// Backward of the selective scan for the layouts the tiled kernel (bwd.cu) does not
// take: the per-head layout (one scalar A, delta row and delta_bias per head) and
// dstate 8, 32, 64 or 128 as well as 16.  The gradients are the ones ssm_scan.h
// states for ssm_selective_scan_bwd (the chain rule through the recurrence; the
// states are recomputed, as the "Agent 229: SSM optimization patterns" page,
// section 4 "Activation Recomputation", describes: checkpoints at chunk
// boundaries, recomputation inside a chunk).  For a per-head shape the head's
// gradients are the sums over its channels: ddelta[b, h, t] and ddelta_bias[h] over
// the channels of head h, dA[h] over its channels and states.
//
// One CTA owns `cpb` channels of one batch row (inside one group) for the whole
// sequence, one thread per (channel, state), up to 256 threads (512 from dstate 64
// on): nothing waits on another CTA.
//   1. A forward pass stores the state at the start of every segment (256 steps)
//      in the workspace.
//   2. Segments are then taken last to first.  A forward pass over the segment
//      keeps the state entering each of its 32-step blocks in shared memory; the
//      blocks are taken last to first: the block's states are recomputed into
//      shared memory, the state gradient g is walked back through the block
//      (g += dy C; keep g; g *= dA), and two passes over shared memory form the
//      sums: over the states of a channel (y, sum g B, the decay term of ddt) for
//      du, ddelta and dz, and over the CTA's channels (g du, dy h) for dB and dC.
// dB, dC and the per-head ddelta are added across CTAs with atomic adds (their last
// bits may differ between calls); a second set of kernels adds the per-row dA, dD
// partials and ddelta into ddelta_bias in a fixed order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "bwd_generic.h"
#include "scan_kernel.cuh"   // ex2_approx, rcp_approx, softplus1, kLog2e

namespace ssm {
namespace {

constexpr int gK = 32;                 // steps per block
constexpr int gSegB = 8;               // blocks per segment
constexpr int gSeg = gK * gSegB;       // steps per segment (a workspace checkpoint each)

struct GParams {
    const void *u, *delta, *z, *dout, *B, *C;
    const float *A, *D, *bias, *h0, *dlast;
    void *du, *dz;
    float *dB, *dC, *dh0;
    float* dd_acc;      // (batch, nheads, L) fp32, zeroed: ddelta summed over a head's channels
    float* dA_part;     // (batch, dim, N): per-row sums of g h_(t-1) dt dA
    float* dD_part;     // (batch, dim): per-row sums of dy u
    float* ckpt;        // (batch, dim, nseg, N): the state entering every segment
    int64_t batch, dim, seqlen, nheads, ngroups;
    int cpb;            // channels per CTA (a power of two dividing dim / ngroups)
    int nseg;           // segments of gSeg steps
    int softplus;
    int head;           // 1: one scalar A per head
    int red_vec;        // dB, dC rows take 16-byte atomic adds (L % 4 == 0, 16-byte aligned)
};

template <typename T> struct GIo;
template <> struct GIo<float> {
    using raw = float;
    __device__ static float f(raw v) { return v; }
    __device__ static float ld(const void* p, int64_t i) { return static_cast<const float*>(p)[i]; }
    __device__ static void st(void* p, int64_t i, float v) { static_cast<float*>(p)[i] = v; }
};
template <> struct GIo<__nv_bfloat16> {
    using raw = unsigned short;
    __device__ static float f(raw v) { return __uint_as_float((uint32_t)v << 16); }
    __device__ static float ld(const void* p, int64_t i) {
        return __uint_as_float((uint32_t) static_cast<const unsigned short*>(p)[i] << 16);
    }
    __device__ static void st(void* p, int64_t i, float v) {
        static_cast<unsigned short*>(p)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
};

__device__ __forceinline__ float gsigmoid(float x) { return rcp_approx(1.f + ex2_approx(x * -kLog2e)); }

__device__ __forceinline__ void gred4(float* dst, const float (&v)[4]) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3])
                 : "memory");
}

// Shared memory (floats) for T = cpb * N threads.  The state and state-gradient rows
// (sH, sG) are T + 1 floats long, so that a thread walking one row and its neighbours
// walking the next meet different banks.  B and C are kept per step, [step][N + 1]: a
// thread reads its own state's column and a team a step's row, both without bank
// conflicts.  The per-(channel, step) arrays are [channel][KP] with KP a multiple of 4:
// a thread reads four steps of its channel in one 16-byte load.
constexpr int KP = gK + 4;
enum { PC_DT = 0, PC_DU, PC_U, PC_X, PC_DY, PC_DOUT, PC_Z, PC_DA, PC_W, kPC };
// PC_DA, PC_W (one A per head): the step's decay dA = exp(dt A) and dt dA, formed once per
// (channel, step) for all of its states
struct GSmem {
    int T, TP, N, NB, cpb, NCH;
    int H, G, BLK, Bs, Cs, PART, PC, DD, KC;   // offsets: sH, sG, sBlk, sB, sC, chunk sums, per-(channel, step) arrays
    int total;
    __host__ __device__ GSmem(int n, int c)
        : T(c * n), TP(c * n + 4), N(n), NB(n + 4), cpb(c), NCH((n + 31) / 32) {
        H = 0;                              // [gK + 1][TP]: the state entering the block, then after each step
        G = H + (gK + 1) * TP;              // [gK][TP]: dLoss/dh_t of each step
        BLK = G + gK * TP;                  // [gSegB][T]: the state entering each block of the segment
        Bs = BLK + gSegB * T;               // [gK][NB]: B of the block
        Cs = Bs + gK * NB;                  // [gK][NB]: C of the block
        PART = Cs + gK * NB;                // [cpb * NCH chunks][3][gK]: a chunk's parts of y, sum g B, the decay term
        PC = (PART + cpb * NCH * 3 * gK + 3) / 4 * 4;   // kPC arrays [cpb][KP], 16-byte aligned
        DD = PC + kPC * cpb * KP;           // [cpb][gK]: a block's ddelta terms (channels of one head)
        KC = DD + cpb * gK;                 // [cpb][4]: per channel A of its head, D, delta_bias of its row
        total = KC + 4 * cpb;
    }
};

// PREF: the CTA holds at least 4 channels (at most 8 B and C values per thread and block),
// so a block's inputs fit in registers and are loaded one block ahead.  HEAD: one scalar A
// per head (the decay of a step is the same for every state of a channel).
template <typename T, int N, bool PREF, bool HEAD>
__global__ void __launch_bounds__(N >= 64 ? 512 : 256) scan_bwd_generic_kernel(const GParams p) {
    extern __shared__ __align__(16) float gsm[];
    const GSmem S(N, p.cpb);
    const int NT = S.T, TP = S.TP;
    constexpr int NB = N + 4;
    const int tid = threadIdx.x;
    const int c = tid / N, n = tid % N;
    const int64_t L = p.seqlen, Dm = p.dim, H = p.nheads, G = p.ngroups;
    const int64_t P = Dm / H;
    const int64_t tiles_per_row = Dm / p.cpb;
    const int64_t b = blockIdx.x / tiles_per_row;
    const int64_t d0 = (blockIdx.x % tiles_per_row) * p.cpb;
    const int64_t d = d0 + c, row = b * Dm + d;
    const int64_t g = d0 / (Dm / G);
    float* sH = gsm + S.H;
    float* sG = gsm + S.G;
    float* sBlk = gsm + S.BLK;
    float* sB = gsm + S.Bs;
    float* sC = gsm + S.Cs;
    float* sPart = gsm + S.PART;
    float* pc = gsm + S.PC;
    float* sDD = gsm + S.DD;
    float* sKc = gsm + S.KC;
    const int cpb = p.cpb;
    auto at = [&](int arr, int cc, int k) -> float& { return pc[(arr * cpb + cc) * KP + k]; };
    auto at4 = [&](int arr, int cc, int k) -> float4 {
        return *reinterpret_cast<const float4*>(pc + (arr * cpb + cc) * KP + k);
    };
    // one A per head with at least 32 states: dA's terms are w_t sum_n g h_(t-1) per (channel,
    // step), the decay sum pass A forms anyway; the (channel, step) threads of pass A add them
    // (one item each: cpb * gK <= cpb * N threads)
    constexpr bool DA_SUM = HEAD && N >= 32;
    // pass B's first thread: past the threads of pass A's second half when half the CTA or
    // more is left for it, so that the two phases overlap instead of queueing on one thread
    const int pb0 = NT >= 2 * cpb * gK ? cpb * gK : 0;
    float da_item = 0.f;
    // every channel of the CTA in one head: the head's ddelta terms are summed here first
    const bool one_head = HEAD && d0 / P == (d0 + cpb - 1) / P;

    // A of this thread's (channel, state), natural units and log2 units
    const float An = HEAD ? __ldg(p.A + d / P) : __ldg(p.A + d * N + n);
    // per-channel constants, read once (the first block's staging follows a barrier)
    for (int cc = tid; cc < cpb; cc += NT) {
        const int64_t dd = d0 + cc, hh = dd / P;
        sKc[cc * 4 + 0] = HEAD ? __ldg(p.A + hh) : 0.f;
        sKc[cc * 4 + 1] = p.D ? __ldg(p.D + dd) : 0.f;
        sKc[cc * 4 + 2] = p.bias ? __ldg(p.bias + hh) : 0.f;
    }
    const float a2 = An * kLog2e;
    const int nblk = (int)((L + gK - 1) / gK);

    // Block blk in two halves: load() reads its inputs into registers (issued a block
    // ahead, so the loads are in flight while the current block runs), store() writes
    // them to shared memory with the per-(channel, step) values: dt and dt*u (full: also
    // u, the softplus argument x, dy = dout silu(z), dout, z; one A per head: dA, dt dA),
    // and the B (full: C) rows.
    constexpr int PPT = gK / N > 0 ? gK / N : 1;   // (channel, step) pairs per thread, at most
    // B and C rows in 16-byte pieces of EPC steps: CPR pieces per row and block, at most VPT
    // per thread (PREF: at least 4 channels, so at least 4 N threads)
    constexpr int EPC = 16 / (int)sizeof(T), CPR = gK / EPC;
    constexpr int VPT = PREF ? (CPR / 4 > 0 ? CPR / 4 : 1) : 1;
    const bool vecbc = ((reinterpret_cast<uintptr_t>(p.B) | reinterpret_cast<uintptr_t>(p.C)) & 15u) == 0 &&
                       L % EPC == 0;
    float ru[PPT], rx[PPT], rdo[PPT], rz[PPT];
    uint4 rb[VPT], rc[VPT];
    // EPC elements of row `src` from step t, zero past L (16-byte load when vecbc and whole)
    auto piece = [&](const void* src, int64_t off, int64_t t) -> uint4 {
        if (vecbc && t + EPC <= L) return __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(src) + off));
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        typename GIo<T>::raw* e = reinterpret_cast<typename GIo<T>::raw*>(&v);
        for (int j = 0; j < EPC; ++j)
            if (t + j < L) e[j] = reinterpret_cast<const typename GIo<T>::raw*>(src)[off + j];
        return v;
    };
    auto load = [&](int blk, bool full) {
        if constexpr (!PREF) return;   // fewer than 4 channels: store() loads for itself
        const int64_t t0 = (int64_t)blk * gK;
#pragma unroll
        for (int e = 0; e < PPT; ++e) {
            const int i = tid + e * NT;
            ru[e] = rx[e] = rdo[e] = rz[e] = 0.f;
            if (i < cpb * gK) {
                const int cc = i / gK, k = i % gK;
                const int64_t t = t0 + k, dd = d0 + cc, hh = dd / P, rr = b * Dm + dd;
                if (t < L) {
                    ru[e] = GIo<T>::ld(p.u, rr * L + t);
                    rx[e] = GIo<T>::ld(p.delta, (b * H + hh) * L + t);   // delta_bias added at staging
                    if (full) {
                        rdo[e] = GIo<T>::ld(p.dout, rr * L + t);
                        if (p.z) rz[e] = GIo<T>::ld(p.z, rr * L + t);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < VPT; ++e) {
            const int i = tid + e * NT;
            if (i < N * CPR) {
                const int nn = i / CPR, q = i % CPR;
                const int64_t t = t0 + q * EPC, off = ((b * G + g) * N + nn) * L + t;
                rb[e] = piece(p.B, off, t);
                if (full) rc[e] = piece(p.C, off, t);
            }
        }
    };
    // the per-(channel, step) values of one pair from its inputs (past L: dt = 0, so dA = 1)
    auto put = [&](int cc, int k, bool valid, float uv, float xd, float dov, float zv, bool full) {
        const float x = xd + sKc[cc * 4 + 2];   // + delta_bias
        const float dt = valid ? (p.softplus ? softplus1(x) : x) : 0.f;
        at(PC_DT, cc, k) = dt;
        at(PC_DU, cc, k) = dt * uv;
        if (HEAD) {
            const float dA = ex2_approx(dt * (sKc[cc * 4 + 0] * kLog2e));
            at(PC_DA, cc, k) = dA;
            at(PC_W, cc, k) = dt * dA;
        }
        if (full) {
            at(PC_U, cc, k) = uv;
            at(PC_X, cc, k) = x;
            at(PC_DY, cc, k) = p.z ? dov * (zv * gsigmoid(zv)) : dov;
            at(PC_DOUT, cc, k) = dov;
            at(PC_Z, cc, k) = zv;
        }
    };
    auto store = [&](int blk, bool full) {
        const int64_t t0 = (int64_t)blk * gK;
        if constexpr (!PREF) {
            // no registers to spare: load and store in one go
            for (int i = tid; i < cpb * gK; i += NT) {
                const int cc = i / gK, k = i % gK;
                const int64_t t = t0 + k, dd = d0 + cc, hh = dd / P, rr = b * Dm + dd;
                float uv = 0.f, x = 0.f, dov = 0.f, zv = 0.f;
                if (t < L) {
                    uv = GIo<T>::ld(p.u, rr * L + t);
                    x = GIo<T>::ld(p.delta, (b * H + hh) * L + t);
                    if (full) {
                        dov = GIo<T>::ld(p.dout, rr * L + t);
                        if (p.z) zv = GIo<T>::ld(p.z, rr * L + t);
                    }
                }
                put(cc, k, t < L, uv, x, dov, zv, full);
            }
            for (int i = tid; i < N * gK; i += NT) {
                const int nn = i / gK, k = i % gK;
                const int64_t t = t0 + k, off = ((b * G + g) * N + nn) * L + t;
                sB[k * NB + nn] = t < L ? GIo<T>::ld(p.B, off) : 0.f;
                if (full) sC[k * NB + nn] = t < L ? GIo<T>::ld(p.C, off) : 0.f;
            }
            return;
        }
#pragma unroll
        for (int e = 0; e < PPT; ++e) {
            const int i = tid + e * NT;
            if (i < cpb * gK) {
                const int cc = i / gK, k = i % gK;
                put(cc, k, t0 + k < L, ru[e], rx[e], rdo[e], rz[e], full);
            }
        }
#pragma unroll
        for (int e = 0; e < VPT; ++e) {
            const int i = tid + e * NT;
            if (i < N * CPR) {
                const int nn = i / CPR, k0 = (i % CPR) * EPC;
                const typename GIo<T>::raw* vb = reinterpret_cast<const typename GIo<T>::raw*>(&rb[e]);
                const typename GIo<T>::raw* vc = reinterpret_cast<const typename GIo<T>::raw*>(&rc[e]);
#pragma unroll
                for (int j = 0; j < EPC; ++j) {
                    sB[(k0 + j) * NB + nn] = GIo<T>::f(vb[j]);
                    if (full) sC[(k0 + j) * NB + nn] = GIo<T>::f(vc[j]);
                }
            }
        }
    };
    // the recurrence over the staged block from state h (steps past L have dt = 0: no
    // change); keep: every state into sH (row 0 the entering state, row k + 1 after step k)
    auto run_block = [&](float h, auto keep_c) -> float {
        constexpr bool keep = decltype(keep_c)::value;   // a compile-time choice: no branch per step
        if (keep) sH[tid] = h;
#pragma unroll 2
        for (int k0 = 0; k0 < gK; k0 += 4) {
            const float4 du4 = at4(PC_DU, c, k0);
            const float4 x4 = HEAD ? at4(PC_DA, c, k0) : at4(PC_DT, c, k0);
            const float duv[4] = {du4.x, du4.y, du4.z, du4.w}, xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = k0 + e;
                const float dA = HEAD ? xv[e] : ex2_approx(xv[e] * a2);
                h = fmaf(dA, h, duv[e] * sB[k * NB + n]);
                if (keep) sH[(k + 1) * TP + tid] = h;
            }
        }
        return h;
    };

    // ---- 1. forward: the state entering every segment, into the workspace
    float h = p.h0 ? __ldg(p.h0 + row * N + n) : 0.f;
    if (nblk > 0) load(0, false);
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk % gSegB == 0) p.ckpt[(row * p.nseg + blk / gSegB) * N + n] = h;
        __syncthreads();   // the previous block is done with the staged arrays
        store(blk, false);
        __syncthreads();
        if (blk + 1 < nblk) load(blk + 1, false);
        h = run_block(h, std::false_type{});
    }

    // ---- 2. segments last to first
    float gst = p.dlast ? __ldg(p.dlast + row * N + n) : 0.f;   // dLoss/dh after the last step
    float da = 0.f, dDacc = 0.f;
    // pass A: a warp per chunk of up to 32 states of one channel, a lane per step
    constexpr int NCH = (N + 31) / 32, NC = N < 32 ? N : 32;
    const int warp = tid / 32, lane = tid % 32, nwarps = NT / 32 > 0 ? NT / 32 : 1;
    // channels of one head: a block's ddelta terms wait in sDD, and after the next barrier a
    // thread per step adds them up and into dd_acc (one atomic add per step)
    int64_t dd_t0 = -1;
    auto flush_dd = [&]() {
        if (one_head && dd_t0 >= 0) {
            for (int k = tid; k < gK && dd_t0 + k < L; k += NT) {   // fewer threads than steps: a loop
                float s = 0.f;
                for (int cc = 0; cc < cpb; ++cc) s += sDD[cc * gK + k];
                atomicAdd(p.dd_acc + (b * H + d0 / P) * L + dd_t0 + k, s);
            }
            dd_t0 = -1;
        }
    };
    for (int seg = p.nseg - 1; seg >= 0; --seg) {
        const int b0 = seg * gSegB, b1 = min(nblk, b0 + gSegB);
        float hs = p.ckpt[(row * p.nseg + seg) * N + n];
        load(b0, false);
        for (int blk = b0; blk < b1; ++blk) {
            sBlk[(blk - b0) * NT + tid] = hs;
            __syncthreads();
            store(blk, false);
            __syncthreads();
            if (blk + 1 < b1) load(blk + 1, false);
            else load(b1 - 1, true);   // the first block of the walk
            hs = run_block(hs, std::false_type{});
        }
        for (int blk = b1 - 1; blk >= b0; --blk) {
            const int64_t t0 = (int64_t)blk * gK;
            __syncthreads();
            flush_dd();   // the previous block's (its terms are in after the barrier)
            store(blk, true);
            __syncthreads();
            if (blk > b0) load(blk - 1, true);
            run_block(sBlk[(blk - b0) * NT + tid], std::true_type{});
            const int kend = (int)(L - t0 < gK ? L - t0 : gK);   // steps of the block inside L
            // the state gradient back through the block: g += dy C is dLoss/dh_t
#pragma unroll 2
            for (int k0 = gK - 4; k0 >= 0; k0 -= 4) {
                const float4 dy4 = at4(PC_DY, c, k0);
                const float4 x4 = HEAD ? at4(PC_DA, c, k0) : at4(PC_DT, c, k0);
                const float4 w4 = HEAD ? at4(PC_W, c, k0) : x4;
                const float dyv[4] = {dy4.x, dy4.y, dy4.z, dy4.w}, xv[4] = {x4.x, x4.y, x4.z, x4.w};
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 3; e >= 0; --e) {
                    const int k = k0 + e;
                    if (k < kend) {
                        gst = fmaf(dyv[e], sC[k * NB + n], gst);
                        sG[k * TP + tid] = gst;
                        float dA, w;
                        if (HEAD) {
                            dA = xv[e];
                            w = wv[e];
                        } else {
                            dA = ex2_approx(xv[e] * a2);
                            w = xv[e] * dA;
                        }
                        if (!DA_SUM) da = fmaf(gst * sH[k * TP + tid], w, da);
                        gst *= dA;
                    } else {
                        sG[k * TP + tid] = 0.f;
                    }
                }
            }
            if (n == 0)
                for (int k = 0; k < gK; ++k)
                    if (k < kend) dDacc = fmaf(at(PC_DY, c, k), at(PC_U, c, k), dDacc);
            __syncthreads();   // sH and sG complete
            // pass A, first half: per chunk and step (lane), the chunk's parts of y = sum C h,
            // gB = sum g B and q = sum g h_(t-1) (A dA) into sPart.  No shuffles: each lane reads
            // its step's rows four states at a time, and rows 4 mod 32 floats apart put the eight
            // lanes of a 16-byte phase in different banks.
            if (NT >= 32) {
                for (int ch = warp; ch < cpb * NCH; ch += nwarps) {
                    const int cc = ch / NCH, n0 = (ch % NCH) * NC, k = lane;
                    const float* grow = sG + k * TP + cc * N + n0;
                    const float* hrow = sH + (k + 1) * TP + cc * N + n0;
                    const float* prow = sH + k * TP + cc * N + n0;
                    const float* brow = sB + k * NB + n0;
                    const float* crow = sC + k * NB + n0;
                    const float dt = at(PC_DT, cc, k);
                    float y = 0.f, gB = 0.f, q = 0.f;
#pragma unroll 2
                    for (int i0 = 0; i0 < NC; i0 += 4) {
                        const float4 g4 = *reinterpret_cast<const float4*>(grow + i0);
                        const float4 h4 = *reinterpret_cast<const float4*>(hrow + i0);
                        const float4 p4 = *reinterpret_cast<const float4*>(prow + i0);
                        const float4 b4 = *reinterpret_cast<const float4*>(brow + i0);
                        const float4 c4 = *reinterpret_cast<const float4*>(crow + i0);
                        const float gv[4] = {g4.x, g4.y, g4.z, g4.w}, hv[4] = {h4.x, h4.y, h4.z, h4.w};
                        const float pv[4] = {p4.x, p4.y, p4.z, p4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
                        const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            y = fmaf(cv[e], hv[e], y);
                            gB = fmaf(gv[e], bv[e], gB);
                            if (HEAD) {
                                q = fmaf(gv[e], pv[e], q);
                            } else {
                                const float Ann = __ldg(p.A + (d0 + cc) * N + n0 + i0 + e);
                                q = fmaf(gv[e] * pv[e], Ann * ex2_approx(dt * (Ann * kLog2e)), q);
                            }
                        }
                    }
                    float* pp = sPart + ch * 3 * gK + k;
                    pp[0] = y;
                    pp[gK] = gB;
                    pp[2 * gK] = q;
                }
            } else {
                // fewer than 32 threads (one channel of dstate 8 or 16): a thread per step
                for (int it = tid; it < cpb * NCH * gK; it += NT) {
                    const int ch = it / gK, k = it % gK, cc = ch / NCH, n0 = (ch % NCH) * NC;
                    const float dt = at(PC_DT, cc, k);
                    float y = 0.f, gB = 0.f, q = 0.f;
                    for (int i = 0; i < NC; ++i) {
                        const float gv = sG[k * TP + cc * N + n0 + i], hp = sH[k * TP + cc * N + n0 + i];
                        y = fmaf(sC[k * NB + n0 + i], sH[(k + 1) * TP + cc * N + n0 + i], y);
                        gB = fmaf(gv, sB[k * NB + n0 + i], gB);
                        if (HEAD) {
                            q = fmaf(gv, hp, q);
                        } else {
                            const float Ann = __ldg(p.A + (d0 + cc) * N + n0 + i);
                            q = fmaf(gv * hp, Ann * ex2_approx(dt * (Ann * kLog2e)), q);
                        }
                    }
                    float* pp = sPart + ch * 3 * gK + k;
                    pp[0] = y;
                    pp[gK] = gB;
                    pp[2 * gK] = q;
                }
            }
            __syncthreads();
            // second half: per (channel, step), the chunks' parts added in order, then the outputs
            for (int it = tid; it < cpb * gK; it += NT) {
                const int cc = it / gK, k = it % gK;
                const int64_t t = t0 + k;
                if (t >= L) continue;
                float y = 0.f, gB = 0.f, q = 0.f;
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
                    const float* pp = sPart + (cc * NCH + j) * 3 * gK + k;
                    y += pp[0];
                    gB += pp[gK];
                    q += pp[2 * gK];
                }
                const float dt = at(PC_DT, cc, k);
                const int64_t dd = d0 + cc, hh = dd / P, rr = b * Dm + dd;
                if (DA_SUM) da_item = fmaf(q, at(PC_W, cc, k), da_item);   // sum_n g h_(t-1) times dt dA
                if (HEAD) q *= sKc[cc * 4 + 0] * at(PC_DA, cc, k);   // one decay for every state
                const float uv = at(PC_U, cc, k), dy = at(PC_DY, cc, k);
                const float Dv = sKc[cc * 4 + 1];
                GIo<T>::st(p.du, rr * L + t, fmaf(dt, gB, dy * Dv));
                const float ddt = fmaf(uv, gB, q);
                const float ddl = p.softplus ? ddt * gsigmoid(at(PC_X, cc, k)) : ddt;
                if (one_head) sDD[cc * gK + k] = ddl;   // summed over the CTA's channels after the next barrier
                else atomicAdd(p.dd_acc + (b * H + hh) * L + t, ddl);
                if (p.z) {
                    const float zv = at(PC_Z, cc, k), sg = gsigmoid(zv);
                    GIo<T>::st(p.dz, rr * L + t, at(PC_DOUT, cc, k) * fmaf(Dv, uv, y) * (sg * fmaf(zv, 1.f - sg, 1.f)));
                }
            }
            dd_t0 = t0;
            // pass B: per (state, step), dB = sum over channels of g dt u, dC = of dy h_t
            // (four consecutive steps per thread: one 16-byte atomic add each for dB and dC;
            // consecutive threads take consecutive states)
            // (where there are threads to spare, not on those that ran pass A's second half)
            for (int i = tid - pb0; i >= 0 && i < N * (gK / 4); i += NT - pb0) {
                const int nn = i % N, k4 = (i / N) * 4;
                if (t0 + k4 >= L) continue;
                float sb[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int cc = 0; cc < cpb; ++cc) {
                    const int idx = cc * N + nn;
                    const float4 du4 = at4(PC_DU, cc, k4), dy4 = at4(PC_DY, cc, k4);
                    const float duv[4] = {du4.x, du4.y, du4.z, du4.w}, dyv[4] = {dy4.x, dy4.y, dy4.z, dy4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = k4 + e;
                        sb[e] = fmaf(sG[k * TP + idx], duv[e], sb[e]);
                        sc[e] = fmaf(dyv[e], sH[(k + 1) * TP + idx], sc[e]);
                    }
                }
                const int64_t off = ((b * G + g) * N + nn) * L + t0 + k4;
                if (p.red_vec && t0 + k4 + 3 < L) {
                    gred4(p.dB + off, sb);
                    gred4(p.dC + off, sc);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (t0 + k4 + e < L) {
                            atomicAdd(p.dB + off + e, sb[e]);
                            atomicAdd(p.dC + off + e, sc[e]);
                        }
                }
            }
        }
    }
    __syncthreads();
    flush_dd();
    if (p.dh0) p.dh0[row * N + n] = gst;
    if constexpr (DA_SUM) {
        // channel cc's total from the gK pass-A threads of warp cc (their items are (cc, step))
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) da_item += __shfl_xor_sync(0xffffffffu, da_item, o);
        p.dA_part[row * N + n] = 0.f;
        __syncthreads();
        if (tid < cpb * gK && lane == 0) p.dA_part[(b * Dm + d0 + tid / gK) * N] = da_item;
    } else {
        p.dA_part[row * N + n] = da;
    }
    if (n == 0) p.dD_part[row] = dDacc;
}

}  // namespace
}  // namespace ssm

namespace ssm {
namespace {

// ddelta in the io dtype from the fp32 sums
template <typename T>
__global__ void __launch_bounds__(256) gbwd_ddelta(const float* acc, void* out, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        GIo<T>::st(out, i, acc[i]);
}

// Per head h (one CTA each, 256 threads, fixed order): ddelta_bias[h] = the sum over
// batch rows and steps of ddelta; with one A per head, dA[h] = the sum of the per-row
// partials of its channels and states.
__global__ void __launch_bounds__(256) gbwd_heads(const float* acc, const float* dA_part, float* dbias, float* dA,
                                                  int64_t batch, int64_t dim, int64_t nheads, int64_t L, int N,
                                                  int head) {
    __shared__ float red[2][256];
    const int64_t h = blockIdx.x;
    const int64_t P = dim / nheads;
    float s0 = 0.f, s1 = 0.f;
    for (int64_t i = threadIdx.x; i < batch * L; i += 256) {
        const int64_t b = i / L, t = i % L;
        s0 += acc[(b * nheads + h) * L + t];
    }
    if (head)
        for (int64_t i = threadIdx.x; i < batch * P * N; i += 256) {
            const int64_t b = i / (P * N), r = i % (P * N);
            s1 += dA_part[(b * dim + h * P) * N + r];
        }
    red[0][threadIdx.x] = s0;
    red[1][threadIdx.x] = s1;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) {
            red[0][threadIdx.x] += red[0][threadIdx.x + o];
            red[1][threadIdx.x] += red[1][threadIdx.x + o];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        if (dbias) dbias[h] = red[0][0];
        if (head) dA[h] = red[1][0];
    }
}

// Per channel (and state): dD[d] and, with A per channel, dA[d][n] as sums over the
// batch rows in order.
__global__ void __launch_bounds__(256) gbwd_rows(const float* dA_part, const float* dD_part, float* dA, float* dD,
                                                 int64_t batch, int64_t dim, int N, int head) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (!head && i < dim * N) {
        float s = 0.f;
        for (int64_t b = 0; b < batch; ++b) s += dA_part[b * dim * N + i];
        dA[i] = s;
    }
    if (dD && i < dim) {
        float s = 0.f;
        for (int64_t b = 0; b < batch; ++b) s += dD_part[b * dim + i];
        dD[i] = s;
    }
}

int64_t align256g(int64_t x) { return (x + 255) / 256 * 256; }

struct GLayout {
    int64_t dd, dA, dD, ck, total;   // byte offsets after the 256-byte header
};

// channels per CTA: the largest power of two up to 256 / N (512 / N from N = 64 on) that divides
// dim / ngroups
int gcpb(const ssm_dims_t& d) {
    const int64_t per_group = d.dim / d.ngroups;
    int c = (d.dstate >= 64 ? 512 : 256) / (int)d.dstate;
    while (c > 1 && per_group % c) c >>= 1;
    return c;
}

GLayout glayout(const ssm_dims_t& d) {
    const int64_t nseg = (d.seqlen + gSeg - 1) / gSeg;
    GLayout w;
    w.dd = 256;
    w.dA = align256g(w.dd + d.batch * d.nheads * d.seqlen * 4);
    w.dD = align256g(w.dA + d.batch * d.dim * d.dstate * 4);
    w.ck = align256g(w.dD + d.batch * d.dim * 4);
    w.total = align256g(w.ck + d.batch * d.dim * nseg * d.dstate * 4);
    return w;
}

template <typename T, int N, bool PREF, bool HEAD>
int glaunch_one(const GParams& prm, unsigned grid, cudaStream_t s) {
    const GSmem S(N, prm.cpb);
    const size_t smem = (size_t)S.total * 4;
    if (smem > 227 * 1024) return SSM_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 && cudaFuncSetAttribute(scan_bwd_generic_kernel<T, N, PREF, HEAD>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    scan_bwd_generic_kernel<T, N, PREF, HEAD><<<grid, (unsigned)S.T, smem, s>>>(prm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
template <typename T, int N>
int glaunch(const GParams& prm, unsigned grid, cudaStream_t s) {
    if (prm.head)
        return prm.cpb >= 4 ? glaunch_one<T, N, true, true>(prm, grid, s) : glaunch_one<T, N, false, true>(prm, grid, s);
    return prm.cpb >= 4 ? glaunch_one<T, N, true, false>(prm, grid, s) : glaunch_one<T, N, false, false>(prm, grid, s);
}

template <typename T>
int glaunch_n(const GParams& prm, int N, unsigned grid, cudaStream_t s) {
    switch (N) {
        case 8: return glaunch<T, 8>(prm, grid, s);
        case 16: return glaunch<T, 16>(prm, grid, s);
        case 32: return glaunch<T, 32>(prm, grid, s);
        case 64: return glaunch<T, 64>(prm, grid, s);
        case 128: return glaunch<T, 128>(prm, grid, s);
        default: return SSM_ERR_UNSUPPORTED;
    }
}

}  // namespace

int bwd_generic_supported(const ssm_dims_t& d) {
    const int64_t N = d.dstate;
    if (N != 8 && N != 16 && N != 32 && N != 64 && N != 128) return SSM_ERR_UNSUPPORTED;
    if (d.batch * (d.dim / gcpb(d)) > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    if (d.batch * d.nheads > 0x7FFFFFFF || d.nheads > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

int64_t bwd_generic_workspace_bytes(const ssm_dims_t& d) { return glayout(d).total; }

int bwd_generic_launch(const ssm_dims_t& d, const void* u, const void* delta, const float* A, const void* B,
                       const void* C, const float* D, const void* z, const float* delta_bias, int softplus,
                       const float* h0, const void* dout, const float* dlast, const ssm_grads_t& gr,
                       unsigned char* ws, cudaStream_t s) {
    const GLayout w = glayout(d);
    GParams prm;
    prm.u = u; prm.delta = delta; prm.z = z; prm.dout = dout; prm.B = B; prm.C = C;
    prm.A = A; prm.D = D; prm.bias = delta_bias; prm.h0 = h0; prm.dlast = dlast;
    prm.du = gr.du; prm.dz = gr.dz; prm.dB = gr.dB; prm.dC = gr.dC; prm.dh0 = gr.dh0;
    prm.dd_acc = reinterpret_cast<float*>(ws + w.dd);
    prm.dA_part = reinterpret_cast<float*>(ws + w.dA);
    prm.dD_part = reinterpret_cast<float*>(ws + w.dD);
    prm.ckpt = reinterpret_cast<float*>(ws + w.ck);
    prm.batch = d.batch; prm.dim = d.dim; prm.seqlen = d.seqlen; prm.nheads = d.nheads; prm.ngroups = d.ngroups;
    prm.cpb = gcpb(d);
    prm.nseg = (int)((d.seqlen + gSeg - 1) / gSeg);
    prm.softplus = softplus ? 1 : 0;
    prm.head = d.nheads != d.dim ? 1 : 0;
    prm.red_vec = d.seqlen % 4 == 0 && ((reinterpret_cast<uintptr_t>(gr.dB) | reinterpret_cast<uintptr_t>(gr.dC)) & 15u) == 0;
    const int64_t N = d.dstate;
    const size_t nbc = (size_t)(d.batch * d.ngroups * N * d.seqlen) * 4;
    // the header (status: nothing here waits, so it stays SSM_OK), the ddelta sums, dB and dC start at zero
    if (cudaMemsetAsync(ws, 0, 8, s) != cudaSuccess ||
        cudaMemsetAsync(ws + w.dd, 0, (size_t)(d.batch * d.nheads * d.seqlen) * 4, s) != cudaSuccess ||
        cudaMemsetAsync(gr.dB, 0, nbc, s) != cudaSuccess || cudaMemsetAsync(gr.dC, 0, nbc, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    const unsigned grid = (unsigned)(d.batch * (d.dim / prm.cpb));
    int rc = d.io_dtype == SSM_BF16 ? glaunch_n<__nv_bfloat16>(prm, (int)N, grid, s)
                                    : glaunch_n<float>(prm, (int)N, grid, s);
    if (rc != SSM_OK) return rc;
    const int64_t ndd = d.batch * d.nheads * d.seqlen;
    const unsigned g1 = (unsigned)((ndd + 255) / 256 < 4096 ? (ndd + 255) / 256 : 4096);
    if (d.io_dtype == SSM_BF16) gbwd_ddelta<__nv_bfloat16><<<g1, 256, 0, s>>>(prm.dd_acc, gr.ddelta, ndd);
    else gbwd_ddelta<float><<<g1, 256, 0, s>>>(prm.dd_acc, gr.ddelta, ndd);
    gbwd_heads<<<(unsigned)d.nheads, 256, 0, s>>>(prm.dd_acc, prm.dA_part, gr.ddelta_bias, gr.dA, d.batch, d.dim,
                                                    d.nheads, d.seqlen, (int)N, prm.head);
    const int64_t nrows = prm.head ? d.dim : d.dim * N;
    gbwd_rows<<<(unsigned)((nrows + 255) / 256), 256, 0, s>>>(prm.dA_part, prm.dD_part, gr.dA, gr.dD, d.batch, d.dim,
                                                              (int)N, prm.head);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace ssm
