// Chunked state-space-dual (SSD) forward on the tensor cores, for the per-head
// layout with a scalar A per head, dstate 128 and head dim 64 (bf16 I/O): the
// "Agent 229: SSM optimization patterns" page, section 2 "Mamba-2 SSD (State
// Space Duality)" (the SSM as a semi-separable matrix, computed in chunks:
// quadratic within a chunk, a recurrence across chunks) and section 9 "Chunked
// Computation"; the result is the same recurrence as the scan kernel's.
//
// One CTA runs one (batch row, head) through its chunks of Q = 128 steps.  With
// a_t = dt_t * A_h * log2(e) and cum the prefix sum of a within the chunk, the
// state H (N x P) at the chunk start, and X, B, C the chunk's u, B, C rows:
//
//   G  = C B^T                                   (Q x Q, K = N)       tensor cores
//   M  = G o [2^(cum_i - cum_j) dt_j]_{j <= i}   (causal decay mask)  threads
//   Y  = M X + diag(2^cum) (C H)                 (Q x P)              tensor cores
//   out = (Y + D x) silu(z)                                           threads
//   B' = B diag(2^(cum_end - cum_j) dt_j)                             threads
//   H  = 2^cum_end H + B'^T X                    (N x P)              tensor cores + threads
//
// Operands the tensor cores read: B, C and X straight from TMA boxes (128-byte
// swizzle; B and C as MN-major tiles, X as K-major), M and B' as K-major tiles
// and H as an MN-major tile written by the threads.  M, B' and H are fp32
// values; each goes in as a bf16 pair hi + lo (lo = the rounding residue), two
// MMAs per product, so the products keep about 16 significant bits: the state
// stays within the fp32 tolerance of the recurrence.  Accumulators live in TMEM:
// G (128 columns), Y (64), C H (64), S (64).
//
// Every wait is bounded (%globaltimer); a wait that runs out records
// SSM_ERR_TIMEOUT and every thread leaves the chunk loop together.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "scan_kernel.cuh"
#include "ssd.h"
#include "tcgen05.cuh"

namespace ssm {
namespace {

constexpr int kQ = 128;     // steps per chunk
constexpr int kP = 64;      // head dim
constexpr int kN = 128;     // state size
constexpr int kThreadsSsd = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0, kColY = 128, kColCH = 192, kColS = 256;

// shared memory (bytes from a 1024-aligned base)
constexpr int OFF_C = 0;                 // C: 2 boxes (t halves) x 128 rows x 128 B
constexpr int OFF_B = 32 * 1024;         // B: same
constexpr int OFF_X = 64 * 1024;         // X (u rows of the head): 2 boxes x 64 rows x 128 B
constexpr int OFF_MB = 80 * 1024;        // M, later B': hi (2 atom columns x 128 rows x 128 B), then lo
constexpr int OFF_H = 144 * 1024;        // H: hi (128 rows x 128 B), then lo
constexpr int OFF_DT = 176 * 1024;       // dt[128] floats, cum[128] floats
constexpr int OFF_BAR = OFF_DT + 1024;   // barriers: full, g, y, s; TMEM base slot
constexpr int kSmemSsd = OFF_BAR + 64 + 1024;   // + slack to align the base up to 1024 bytes
constexpr uint32_t kTxBytes = 2 * 16384 + 2 * 16384 + 2 * 8192;

__device__ __forceinline__ uint32_t bf16_bits(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// v as bf16 hi + bf16 lo (lo = bf16 of the residue)
__device__ __forceinline__ void split2(float v, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi = (uint32_t)__bfloat16_as_ushort(h);
    lo = bf16_bits(v - __bfloat162float(h));
}

// 8 consecutive columns c0..c0+7 of row r of a 128-byte-swizzled tile, as hi and lo pairs
__device__ __forceinline__ void store_pair8(unsigned char* hi_tile, unsigned char* lo_tile, uint32_t r, uint32_t c0,
                                            const float (&v)[8]) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t h0, l0, h1, l1;
        split2(v[2 * q], h0, l0);
        split2(v[2 * q + 1], h1, l1);
        h[q] = h0 | (h1 << 16);
        l[q] = l0 | (l1 << 16);
    }
    const uint32_t off = tc::sw128_off(r, c0);
    *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ float bf16_at(const unsigned char* tile, uint32_t r, uint32_t c) {
    return __bfloat162float(__ushort_as_bfloat16(*reinterpret_cast<const unsigned short*>(tile + tc::sw128_off(r, c))));
}

__global__ void __launch_bounds__(kThreadsSsd, 1) ssd_fwd_kernel(const SsdParams p, const __grid_constant__ SsdMaps m) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* full = bars + 0;
    uint64_t* mb_g = bars + 1;
    uint64_t* mb_y = bars + 2;
    uint64_t* mb_s = bars + 3;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 32);
    float* sdt = reinterpret_cast<float*>(smem + OFF_DT);
    float* scum = sdt + kQ;
    unsigned char* sC = smem + OFF_C;
    unsigned char* sB = smem + OFF_B;
    unsigned char* sX = smem + OFF_X;
    unsigned char* sMhi = smem + OFF_MB;
    unsigned char* sMlo = smem + OFF_MB + 32 * 1024;
    unsigned char* sHhi = smem + OFF_H;
    unsigned char* sHlo = smem + OFF_H + 16 * 1024;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t row = (uint32_t)(32 * quarter + lane);   // this thread's TMEM lane
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / p.nheads, h = bh % p.nheads;
    const int64_t G = p.ngroups, g = h / (p.nheads / G);
    const int64_t L = p.seqlen, Dm = p.dim;
    const int64_t d0 = h * kP;   // first channel of the head
    const uint64_t budget = (uint64_t)p.spin_limit * 256ull;
    const float Ah = __ldg(p.A + h) * kLog2e;
    const float bias = p.bias ? __ldg(p.bias + h) : 0.f;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::alloc(tslot, kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t trow = tbase + ((uint32_t)(32 * quarter) << 16);

    // the state of this thread's row n = row, head-dim half [32*half, 32*half + 32)
    float H[32];
    const bool have_h0 = p.h0 != nullptr;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const int64_t d = d0 + 32 * half + k;
        H[k] = have_h0 ? __ldg(p.h0 + (b * Dm + d) * kN + row) : 0.f;
    }
    if (have_h0) {
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = H[k + e];
            store_pair8(sHhi, sHlo, row, (uint32_t)(32 * half + k), v);
        }
    }
    tc::fence_async_smem();

    const int nchunks = (int)(L / kQ);
    bool failed = false;
    uint64_t* last_bar = nullptr;   // thread 0: the barrier of its latest commit and that phase
    unsigned last_ph = 0;
    for (int c = 0; c < nchunks; ++c) {
        const int64_t t0 = (int64_t)c * kQ;
        const unsigned ph = (unsigned)c & 1u;
        __syncthreads();   // the previous chunk is done with every shared tile
        if (tid == 0) {
            mbar_arrive_tx(full, kTxBytes);
            for (int hb = 0; hb < 2; ++hb) {
                const int x = (int)(t0 + 64 * hb);
                tma_2d(sC + hb * 16384, &m.C, x, (int)((b * G + g) * kN), full);
                tma_2d(sB + hb * 16384, &m.B, x, (int)((b * G + g) * kN), full);
                tma_2d(sX + hb * 8192, &m.u, x, (int)(b * Dm + d0), full);
            }
        }
        // dt and the decay prefix of the chunk (warp 0, four steps per lane)
        if (warp == 0) {
            const unsigned short* drow =
                reinterpret_cast<const unsigned short*>(p.delta) + (b * p.nheads + h) * L + t0 + 4 * lane;
            const uint2 raw = *reinterpret_cast<const uint2*>(drow);
            const uint32_t w2[2] = {raw.x, raw.y};
            float dt[4], pre[4], run = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t bits = (e & 1) ? (w2[e >> 1] & 0xFFFF0000u) : (w2[e >> 1] << 16);
                const float x = __uint_as_float(bits) + bias;
                dt[e] = p.softplus ? softplus1(x) : x;
                run += dt[e] * Ah;
                pre[e] = run;
            }
            float incl = run;   // inclusive scan of the lane totals
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const float base = incl - run;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sdt[4 * lane + e] = dt[e];
                scum[4 * lane + e] = base + pre[e];
            }
        }
        const bool ok_full = mbar_wait(full, ph, budget, p.status);
        if (__syncthreads_or(!ok_full)) { failed = true; break; }   // also publishes dt and cum

        // ---- G = C B^T: M = t (MN-major C tile), N = t (MN-major B tile), K = n
        if (tid == 0) {
            tc::fence_after();
            constexpr uint32_t id = tc::idesc_bf16(128, 128, true, true);
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk) {
                const uint64_t a = tc::desc(sC + kk * 2048, 16384, 1024, tc::kSwizzle128);
                const uint64_t bb = tc::desc(sB + kk * 2048, 16384, 1024, tc::kSwizzle128);
                tc::mma_bf16(tbase + kColG, a, bb, id, kk > 0 ? 1u : 0u);
            }
            tc::commit(mb_g);
            last_bar = mb_g;
            last_ph = ph;
        }
        const bool ok_g = mbar_wait(mb_g, ph, budget, p.status);
        if (__syncthreads_or(!ok_g)) { failed = true; break; }
        tc::fence_after();

        // ---- M = G o decay mask (row i = row, columns j in this thread's half)
        {
            uint32_t g0[32], g1[32];
            tc::ld32(trow + kColG + 64 * half, g0);
            tc::ld32(trow + kColG + 64 * half + 32, g1);
            tc::wait_ld();
            tc::after_wait(g0);
            tc::after_wait(g1);
            const float ci = scum[row];
#pragma unroll
            for (int k = 0; k < 64; k += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = (uint32_t)(64 * half + k + e);
                    const float gv = __uint_as_float(k + e < 32 ? g0[k + e] : g1[k + e - 32]);
                    v[e] = j <= row ? gv * ex2_approx(ci - scum[j]) * sdt[j] : 0.f;
                }
                store_pair8(sMhi + half * 16384, sMlo + half * 16384, row, (uint32_t)k, v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();

        // ---- Y = M X (K-major, K = j) and C H (MN-major, K = n)
        const bool with_state = c > 0 || have_h0;
        if (tid == 0) {
            tc::fence_after();
            constexpr uint32_t idy = tc::idesc_bf16(128, kP, false, false);
            constexpr uint32_t idh = tc::idesc_bf16(128, kP, true, true);
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk) {
                const int at = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t bx = tc::desc(sX + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, tc::kSwizzle128);
                tc::mma_bf16(tbase + kColY, tc::desc(sMhi + at, 16, 1024, tc::kSwizzle128), bx, idy, kk > 0 ? 1u : 0u);
                tc::mma_bf16(tbase + kColY, tc::desc(sMlo + at, 16, 1024, tc::kSwizzle128), bx, idy, 1u);
            }
            if (with_state) {
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint64_t a = tc::desc(sC + kk * 2048, 16384, 1024, tc::kSwizzle128);
                    tc::mma_bf16(tbase + kColCH, a, tc::desc(sHhi + kk * 2048, 16384, 1024, tc::kSwizzle128), idh,
                                 kk > 0 ? 1u : 0u);
                    tc::mma_bf16(tbase + kColCH, a, tc::desc(sHlo + kk * 2048, 16384, 1024, tc::kSwizzle128), idh, 1u);
                }
            }
            tc::commit(mb_y);
            last_bar = mb_y;
            last_ph = ph;
        }
        const bool ok_y = mbar_wait(mb_y, ph, budget, p.status);
        if (__syncthreads_or(!ok_y)) { failed = true; break; }
        tc::fence_after();

        // ---- outputs of step i = row, channels p in this thread's half
        {
            uint32_t yv[32], cv[32];
            tc::ld32(trow + kColY + 32 * half, yv);
            if (with_state) tc::ld32(trow + kColCH + 32 * half, cv);
            tc::wait_ld();
            tc::after_wait(yv);
            if (with_state) tc::after_wait(cv);
            const float e = with_state ? ex2_approx(scum[row]) : 0.f;
            const int64_t t = t0 + row;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const uint32_t pp = (uint32_t)(32 * half + k);
                const int64_t d = d0 + pp;
                const float x = bf16_at(sX + (row >> 6) * 8192, pp, row & 63u);
                float v = __uint_as_float(yv[k]);
                if (with_state) v = fmaf(e, __uint_as_float(cv[k]), v);
                v = fmaf(p.D ? __ldg(p.D + d) : 0.f, x, v);
                const int64_t o = (b * Dm + d) * L + t;
                if (p.z) v *= silu1(__bfloat162float(p.z[o]));
                p.out[o] = __float2bfloat16_rn(v);
            }
        }
        // ---- B' = B diag(2^(cum_end - cum_j) dt_j): row n = row, columns j in this thread's half
        {
            const float cend = scum[kQ - 1];
#pragma unroll
            for (int k = 0; k < 64; k += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = (uint32_t)(64 * half + k + e);
                    v[e] = bf16_at(sB + half * 16384, row, (uint32_t)(k + e)) * ex2_approx(cend - scum[j]) * sdt[j];
                }
                store_pair8(sMhi + half * 16384, sMlo + half * 16384, row, (uint32_t)k, v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();

        // ---- S = B'^T X: M = n (K-major B' tile), N = p (K-major X tile), K = j
        if (tid == 0) {
            tc::fence_after();
            constexpr uint32_t ids = tc::idesc_bf16(128, kP, false, false);
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk) {
                const int at = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t bx = tc::desc(sX + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, tc::kSwizzle128);
                tc::mma_bf16(tbase + kColS, tc::desc(sMhi + at, 16, 1024, tc::kSwizzle128), bx, ids, kk > 0 ? 1u : 0u);
                tc::mma_bf16(tbase + kColS, tc::desc(sMlo + at, 16, 1024, tc::kSwizzle128), bx, ids, 1u);
            }
            tc::commit(mb_s);
            last_bar = mb_s;
            last_ph = ph;
        }
        const bool ok_s = mbar_wait(mb_s, ph, budget, p.status);
        if (__syncthreads_or(!ok_s)) { failed = true; break; }
        tc::fence_after();

        // ---- H = 2^cum_end H + S (row n = row, channels in this thread's half)
        {
            uint32_t sv[32];
            tc::ld32(trow + kColS + 32 * half, sv);
            tc::wait_ld();
            tc::after_wait(sv);
            const float dec = ex2_approx(scum[kQ - 1]);
#pragma unroll
            for (int k = 0; k < 32; ++k) H[k] = fmaf(dec, H[k], __uint_as_float(sv[k]));
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = H[k + e];
                store_pair8(sHhi, sHlo, row, (uint32_t)(32 * half + k), v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
    }
    if (!failed && p.last_state) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const int64_t d = d0 + 32 * half + k;
            p.last_state[(b * Dm + d) * kN + row] = H[k];
        }
    }
    // release TMEM once nothing can still be writing it (a failed chunk may have
    // left tensor-core work in flight: wait, bounded, for every barrier it committed)
    if (failed && tid == 0 && last_bar) mbar_wait(last_bar, last_ph, budget, p.status);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tbase, kTmemCols);
}

}  // namespace

bool ssd_eligible(const ssm_dims_t& d) {
    return d.io_dtype == SSM_BF16 && d.nheads != d.dim && d.dim / d.nheads == kP && d.dstate == kN &&
           d.seqlen >= kQ && d.seqlen % kQ == 0 && d.nheads % d.ngroups == 0 && d.batch * d.nheads <= 0x7FFFFFFF;
}

int ssd_smem_bytes() { return kSmemSsd; }

int ssd_launch(const SsdParams& prm, const SsdMaps& maps, int64_t grid, cudaStream_t s) {
    static const bool attr = cudaFuncSetAttribute(ssd_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  kSmemSsd) == cudaSuccess;
    if (!attr) return SSM_ERR_CUDA;
    if (grid <= 0) return SSM_OK;
    ssd_fwd_kernel<<<(unsigned)grid, kThreadsSsd, kSmemSsd, s>>>(prm, maps);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace ssm
