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
    __device__ static float ld(const void* p, int64_t i) { return static_cast<const float*>(p)[i]; }
    __device__ static void st(void* p, int64_t i, float v) { static_cast<float*>(p)[i] = v; }
};
template <> struct GIo<__nv_bfloat16> {
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

// Shared memory (floats) for T = cpb * N threads; rows of T + 1 floats so that a
// thread walking one row of states and its neighbours walking the next rows meet
// different banks.
struct GSmem {
    int T, TP, N, cpb;
    int H, G, BLK, Bs, Cs, PC;   // offsets: sH, sG, sBlk, sB, sC, per-(channel, step) arrays
    int total;
    __host__ __device__ GSmem(int n, int c) : T(c * n), TP(c * n + 1), N(n), cpb(c) {
        H = 0;                              // [gK + 1][TP]: the state entering the block, then after each step
        G = H + (gK + 1) * TP;              // [gK][TP]: dLoss/dh_t of each step
        BLK = G + gK * TP;                  // [gSegB][T]: the state entering each block of the segment
        Bs = BLK + gSegB * T;               // [N][gK + 1]: B of the block
        Cs = Bs + N * (gK + 1);             // [N][gK + 1]: C of the block
        PC = Cs + N * (gK + 1);             // 7 arrays [cpb][gK + 1]: dt, dt*u, u, x, dy, dout, z
        total = PC + 7 * cpb * (gK + 1);
    }
};
enum { PC_DT = 0, PC_DU, PC_U, PC_X, PC_DY, PC_DOUT, PC_Z };

// PREF: the CTA holds at least 4 channels (at most 8 B and C values per thread and block),
// so a block's inputs fit in registers and are loaded one block ahead
template <typename T, int N, bool PREF>
__global__ void __launch_bounds__(N >= 64 ? 512 : 256) scan_bwd_generic_kernel(const GParams p) {
    extern __shared__ float gsm[];
    const GSmem S(N, p.cpb);
    const int NT = S.T, TP = S.TP;
    constexpr int KP = gK + 1;
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
    float* pc = gsm + S.PC;
    const int cpb = p.cpb;
    auto at = [&](int arr, int cc, int k) -> float& { return pc[(arr * cpb + cc) * KP + k]; };

    // A of this thread's (channel, state), natural units and log2 units
    const float An = p.head ? __ldg(p.A + d / P) : __ldg(p.A + d * N + n);
    const float a2 = An * kLog2e;
    const int nblk = (int)((L + gK - 1) / gK);

    // Block blk in two halves: load() reads its inputs into registers (issued a block
    // ahead, so the loads are in flight while the current block runs), store() writes
    // them to shared memory with the per-(channel, step) values: dt and dt*u (full: also
    // u, the softplus argument x, dy = dout silu(z), dout, z), and the B (full: C) rows.
    constexpr int PPT = gK / N > 0 ? gK / N : 1;   // (channel, step) pairs per thread, at most
    constexpr int BPT = PREF ? 8 : 1;               // B (C) values per thread, at most
    float ru[PPT], rx[PPT], rdo[PPT], rz[PPT], rb[BPT], rc[BPT];
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
                    rx[e] = GIo<T>::ld(p.delta, (b * H + hh) * L + t) + (p.bias ? __ldg(p.bias + hh) : 0.f);
                    if (full) {
                        rdo[e] = GIo<T>::ld(p.dout, rr * L + t);
                        if (p.z) rz[e] = GIo<T>::ld(p.z, rr * L + t);
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < BPT; ++e) {
            const int i = tid + e * NT;
            rb[e] = rc[e] = 0.f;
            if (i < N * gK) {
                const int nn = i / gK, k = i % gK;
                const int64_t t = t0 + k, off = ((b * G + g) * N + nn) * L + t;
                if (t < L) {
                    rb[e] = GIo<T>::ld(p.B, off);
                    if (full) rc[e] = GIo<T>::ld(p.C, off);
                }
            }
        }
    };
    auto store = [&](int blk, bool full) {
        const int64_t t0 = (int64_t)blk * gK;
        if constexpr (!PREF) {
            // no registers to spare: load and store in one go
            for (int i = tid; i < cpb * gK; i += NT) {
                const int cc = i / gK, k = i % gK;
                const int64_t t = t0 + k, dd = d0 + cc, hh = dd / P, rr = b * Dm + dd;
                float dt = 0.f, uv = 0.f, x = 0.f, dov = 0.f, zv = 0.f;
                if (t < L) {
                    uv = GIo<T>::ld(p.u, rr * L + t);
                    x = GIo<T>::ld(p.delta, (b * H + hh) * L + t) + (p.bias ? __ldg(p.bias + hh) : 0.f);
                    dt = p.softplus ? softplus1(x) : x;
                    if (full) {
                        dov = GIo<T>::ld(p.dout, rr * L + t);
                        if (p.z) zv = GIo<T>::ld(p.z, rr * L + t);
                    }
                }
                at(PC_DT, cc, k) = dt;
                at(PC_DU, cc, k) = dt * uv;
                if (full) {
                    at(PC_U, cc, k) = uv;
                    at(PC_X, cc, k) = x;
                    at(PC_DY, cc, k) = p.z ? dov * (zv * gsigmoid(zv)) : dov;
                    at(PC_DOUT, cc, k) = dov;
                    at(PC_Z, cc, k) = zv;
                }
            }
            for (int i = tid; i < N * gK; i += NT) {
                const int nn = i / gK, k = i % gK;
                const int64_t t = t0 + k, off = ((b * G + g) * N + nn) * L + t;
                sB[nn * KP + k] = t < L ? GIo<T>::ld(p.B, off) : 0.f;
                if (full) sC[nn * KP + k] = t < L ? GIo<T>::ld(p.C, off) : 0.f;
            }
            return;
        }
#pragma unroll
        for (int e = 0; e < PPT; ++e) {
            const int i = tid + e * NT;
            if (i < cpb * gK) {
                const int cc = i / gK, k = i % gK;
                const bool valid = t0 + k < L;   // past L: no step (dt = 0)
                const float dt = valid ? (p.softplus ? softplus1(rx[e]) : rx[e]) : 0.f;
                at(PC_DT, cc, k) = dt;
                at(PC_DU, cc, k) = dt * ru[e];
                if (full) {
                    at(PC_U, cc, k) = ru[e];
                    at(PC_X, cc, k) = rx[e];
                    at(PC_DY, cc, k) = p.z ? rdo[e] * (rz[e] * gsigmoid(rz[e])) : rdo[e];
                    at(PC_DOUT, cc, k) = rdo[e];
                    at(PC_Z, cc, k) = rz[e];
                }
            }
        }
#pragma unroll
        for (int e = 0; e < BPT; ++e) {
            const int i = tid + e * NT;
            if (i < N * gK) {
                const int nn = i / gK, k = i % gK;
                sB[nn * KP + k] = rb[e];
                if (full) sC[nn * KP + k] = rc[e];
            }
        }
    };
    // the recurrence over the staged block from state h (steps past L have dt = 0: no
    // change); keep: every state into sH (row 0 the entering state, row k + 1 after step k)
    auto run_block = [&](float h, bool keep) -> float {
        if (keep) sH[tid] = h;
        for (int k = 0; k < gK; ++k) {
            const float dA = ex2_approx(at(PC_DT, c, k) * a2);
            h = fmaf(dA, h, at(PC_DU, c, k) * sB[n * KP + k]);
            if (keep) sH[(k + 1) * TP + tid] = h;
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
        h = run_block(h, false);
    }

    // ---- 2. segments last to first
    float gst = p.dlast ? __ldg(p.dlast + row * N + n) : 0.f;   // dLoss/dh after the last step
    float da = 0.f, dDacc = 0.f;
    // pass A: one team of TS consecutive threads per (channel, step) sums over the states
    constexpr int TS = N > gK ? N / gK : 1;
    const int team = tid / TS, tl = tid % TS, nteams = NT / TS;
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
            hs = run_block(hs, false);
        }
        for (int blk = b1 - 1; blk >= b0; --blk) {
            const int64_t t0 = (int64_t)blk * gK;
            __syncthreads();
            store(blk, true);
            __syncthreads();
            if (blk > b0) load(blk - 1, true);
            run_block(sBlk[(blk - b0) * NT + tid], true);
            // the state gradient back through the block: g += dy C is dLoss/dh_t
            for (int k = gK - 1; k >= 0; --k) {
                if (t0 + k < L) {
                    gst = fmaf(at(PC_DY, c, k), sC[n * KP + k], gst);
                    sG[k * TP + tid] = gst;
                    const float dt = at(PC_DT, c, k);
                    const float dA = ex2_approx(dt * a2);
                    da = fmaf(gst * sH[k * TP + tid], dt * dA, da);
                    gst *= dA;
                } else {
                    sG[k * TP + tid] = 0.f;
                }
            }
            if (n == 0)
                for (int k = 0; k < gK; ++k)
                    if (t0 + k < L) dDacc = fmaf(at(PC_DY, c, k), at(PC_U, c, k), dDacc);
            __syncthreads();   // sH and sG complete
            // pass A: per (channel, step), y = sum C h, gB = sum g B, q = sum g h_(t-1) A dA
            for (int pr = team; pr < cpb * gK; pr += nteams) {
                const int cc = pr / gK, k = pr % gK;
                const int64_t t = t0 + k;
                const float dt = at(PC_DT, cc, k);
                const float dAh = ex2_approx(dt * a2);   // one A per head: the decay of every state
                float y = 0.f, gB = 0.f, q = 0.f;
                for (int nn = tl; nn < N; nn += TS) {
                    const int idx = cc * N + nn;
                    const float gv = sG[k * TP + idx];
                    const float Ann = p.head ? An : __ldg(p.A + (d0 + cc) * N + nn);
                    const float dA = p.head ? dAh : ex2_approx(dt * (Ann * kLog2e));
                    y = fmaf(sC[nn * KP + k], sH[(k + 1) * TP + idx], y);
                    gB = fmaf(gv, sB[nn * KP + k], gB);
                    q = fmaf(gv * sH[k * TP + idx], Ann * dA, q);
                }
#pragma unroll
                for (int o = 1; o < TS; o <<= 1) {
                    y += __shfl_xor_sync(0xffffffffu, y, o);
                    gB += __shfl_xor_sync(0xffffffffu, gB, o);
                    q += __shfl_xor_sync(0xffffffffu, q, o);
                }
                if (tl == 0 && t < L) {
                    const int64_t dd = d0 + cc, hh = dd / P, rr = b * Dm + dd;
                    const float uv = at(PC_U, cc, k), dy = at(PC_DY, cc, k);
                    const float Dv = p.D ? __ldg(p.D + dd) : 0.f;
                    GIo<T>::st(p.du, rr * L + t, fmaf(dt, gB, dy * Dv));
                    const float ddt = fmaf(uv, gB, q);
                    atomicAdd(p.dd_acc + (b * H + hh) * L + t, p.softplus ? ddt * gsigmoid(at(PC_X, cc, k)) : ddt);
                    if (p.z) {
                        const float zv = at(PC_Z, cc, k), sg = gsigmoid(zv);
                        GIo<T>::st(p.dz, rr * L + t, at(PC_DOUT, cc, k) * fmaf(Dv, uv, y) * (sg * fmaf(zv, 1.f - sg, 1.f)));
                    }
                }
            }
            // pass B: per (state, step), dB = sum over channels of g dt u, dC = of dy h_t
            // (four consecutive steps per thread: one 16-byte atomic add each for dB and dC)
            for (int i = tid; i < N * (gK / 4); i += NT) {
                const int nn = i / (gK / 4), k4 = (i % (gK / 4)) * 4;
                if (t0 + k4 >= L) continue;
                float sb[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int cc = 0; cc < cpb; ++cc) {
                    const int idx = cc * N + nn;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = k4 + e;
                        sb[e] = fmaf(sG[k * TP + idx], at(PC_DU, cc, k), sb[e]);
                        sc[e] = fmaf(at(PC_DY, cc, k), sH[(k + 1) * TP + idx], sc[e]);
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
    if (p.dh0) p.dh0[row * N + n] = gst;
    p.dA_part[row * N + n] = da;
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

template <typename T, int N, bool PREF>
int glaunch_one(const GParams& prm, unsigned grid, cudaStream_t s) {
    const GSmem S(N, prm.cpb);
    const size_t smem = (size_t)S.total * 4;
    if (smem > 227 * 1024) return SSM_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 && cudaFuncSetAttribute(scan_bwd_generic_kernel<T, N, PREF>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SSM_ERR_CUDA;
    scan_bwd_generic_kernel<T, N, PREF><<<grid, (unsigned)S.T, smem, s>>>(prm);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
template <typename T, int N>
int glaunch(const GParams& prm, unsigned grid, cudaStream_t s) {
    return prm.cpb >= 4 ? glaunch_one<T, N, true>(prm, grid, s) : glaunch_one<T, N, false>(prm, grid, s);
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
