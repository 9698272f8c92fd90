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
//   X' = diag(w) X,  w_j = 2^(cum_end - cum_j) dt_j                   threads
//   H  = 2^cum_end H + B^T X'                    (N x P)              tensor cores + threads
//
// The output tile of a chunk is written by the threads over the z tile (each thread
// writes out(p, t) where it read z(p, t)) and leaves by a TMA store.
//
// Operands the tensor cores read: B, C and X straight from TMA boxes (128-byte
// swizzle; B and C as MN-major tiles for G and C H, B as a K-major tile for S,
// X K-major), M and X' as K-major tiles and H as an MN-major tile written by the
// threads.  M, X' and H are fp32 values; each goes in as a bf16 pair hi + lo (lo = the rounding residue), two
// MMAs per product, so the products keep about 16 significant bits: the state
// stays within the fp32 tolerance of the recurrence.  Accumulators live in TMEM:
// G (128 columns), Y (64), C H (64), S (64).
//
// Every wait is bounded (%globaltimer); a wait that runs out records
// SSM_ERR_TIMEOUT, and at the next CTA-wide vote (three per chunk) every thread
// leaves the chunk loop together.  Threads wait for the tensor cores' results
// themselves (tcgen05.commit -> mbarrier), without a CTA barrier.
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
constexpr int kThreadsSsd = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0, kColY = 128, kColCH = 192, kColS = 256;

// shared memory (bytes from a 1024-aligned base)
constexpr int OFF_C = 0;                 // C: 2 boxes (t halves) x 128 rows x 128 B
constexpr int OFF_B = 32 * 1024;         // B: same
constexpr int OFF_X = 64 * 1024;         // X (u rows of the head): 2 boxes x 64 rows x 128 B
constexpr int OFF_MB = 80 * 1024;        // M (hi: 2 atom columns x 128 rows x 128 B, then lo), later X' (hi, lo)
constexpr int OFF_H = 144 * 1024;        // H: hi (128 rows x 128 B), then lo
constexpr int OFF_Z = 176 * 1024;        // z (gate rows of the head): 2 boxes x 64 rows x 128 B
constexpr int OFF_DT = 192 * 1024;       // two chunks' dt[128], cum[128], w[128] floats
constexpr int kDec = 3 * kQ;             // floats of one chunk's decay vectors
constexpr int OFF_BAR = OFF_DT + 2 * kDec * 4;   // barriers: full (C, B), full (X), g, y, s; TMEM base slot
constexpr int kSmemSsd = OFF_BAR + 128 + 1024;   // + slack to align the base up to 1024 bytes
constexpr uint32_t kTxCB = 2 * 16384 + 2 * 16384;
constexpr uint32_t kTxX = 2 * 8192;   // X, and as much again for z when there is a gate

// 8 consecutive columns c0..c0+7 of row r of a 128-byte-swizzled tile, as hi and lo
// pairs; the conversions go two values at a time (cvt.rn.bf16x2.f32)
__device__ __forceinline__ void store_pair8(unsigned char* hi_tile, unsigned char* lo_tile, uint32_t r, uint32_t c0,
                                            const float (&v)[8]) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(v[2 * q] - hf.x, v[2 * q + 1] - hf.y);
        h[q] = *reinterpret_cast<const uint32_t*>(&hb);
        l[q] = *reinterpret_cast<const uint32_t*>(&lb);
    }
    const uint32_t off = tc::sw128_off(r, c0);
    *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ float bf16_at(const unsigned char* tile, uint32_t r, uint32_t c) {
    return __bfloat162float(__ushort_as_bfloat16(*reinterpret_cast<const unsigned short*>(tile + tc::sw128_off(r, c))));
}

// The decay vectors of one chunk from its delta bits (delta_bits: four steps per lane of one warp):
// dt, the prefix cum (log2 units), and w = 2^(cum_end - cum) dt, the weight of each
// step's input in the chunk's final state (at most dt, since cum only falls).
__device__ __forceinline__ uint2 delta_bits(const SsdParams& p, int64_t b, int64_t h, int64_t t0, int lane) {
    return __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const unsigned short*>(p.delta) +
                                                (b * p.nheads + h) * p.seqlen + t0 + 4 * lane));
}
__device__ __forceinline__ void chunk_decay(const SsdParams& p, uint2 raw, float Ah, float bias, int lane, float* sdt,
                                            float* scum, float* sw) {
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
    const float cend = __shfl_sync(0xffffffffu, incl, 31);
    float cm[4], wv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        cm[e] = base + pre[e];
        wv[e] = ex2_approx(cend - cm[e]) * dt[e];
    }
    *reinterpret_cast<float4*>(sdt + 4 * lane) = make_float4(dt[0], dt[1], dt[2], dt[3]);
    *reinterpret_cast<float4*>(scum + 4 * lane) = make_float4(cm[0], cm[1], cm[2], cm[3]);
    *reinterpret_cast<float4*>(sw + 4 * lane) = make_float4(wv[0], wv[1], wv[2], wv[3]);
}

// TMA store of a 2-D box from shared memory; bulk-group completion
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
                 "r"(y), "r"(tc::smem_addr(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the committed stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// the committed stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 8 consecutive floats from shared memory (16-byte aligned)
__device__ __forceinline__ void lds8f(const float* src, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 q = *reinterpret_cast<const float4*>(src + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = q.x; v[5] = q.y; v[6] = q.z; v[7] = q.w;
}

// Thread (lane group q = warp % 4, part = warp / 4): TMEM lane / tile row
// row = 32 q + lane, and the part-th quarter of that row's columns (32 of the
// 128 steps j; 16 of the 64 head channels p).
__global__ void __launch_bounds__(kThreadsSsd, 1) ssd_fwd_kernel(const SsdParams p, const __grid_constant__ SsdMaps m) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* full_cb = bars + 0;   // C and B tiles of a chunk
    uint64_t* full_x = bars + 1;    // X tile of a chunk
    uint64_t* mb_g = bars + 2;
    uint64_t* mb_y = bars + 3;
    uint64_t* mb_s = bars + 4;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 64);
    float* sdec = reinterpret_cast<float*>(smem + OFF_DT);   // [2][dt[128], cum[128], w[128]]
    unsigned char* sC = smem + OFF_C;
    unsigned char* sB = smem + OFF_B;
    unsigned char* sX = smem + OFF_X;
    unsigned char* sMhi = smem + OFF_MB;
    unsigned char* sMlo = smem + OFF_MB + 32 * 1024;
    unsigned char* sHhi = smem + OFF_H;
    unsigned char* sHlo = smem + OFF_H + 16 * 1024;
    unsigned char* sZ = smem + OFF_Z;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, part = warp >> 2;
    const uint32_t row = (uint32_t)(32 * quarter + lane);
    const uint32_t j0 = (uint32_t)(32 * part);   // this thread's steps j0 .. j0+31
    const uint32_t p0 = (uint32_t)(16 * part);   // this thread's channels p0 .. p0+15
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / p.nheads, h = bh % p.nheads;
    const int64_t G = p.ngroups, g = h / (p.nheads / G);
    const int64_t L = p.seqlen, Dm = p.dim;
    const int64_t d0 = h * kP;
    const uint64_t budget = (uint64_t)p.spin_limit * 256ull;
    const float Ah = __ldg(p.A + h) * kLog2e;
    const float bias = p.bias ? __ldg(p.bias + h) : 0.f;
    const int bc_row = (int)((b * G + g) * kN);
    const int x_row = (int)(b * Dm + d0);
    const bool gate = p.z != nullptr;
    const uint32_t tx_x = gate ? 2 * kTxX : kTxX;
    const int nchunks = (int)(L / kQ);

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::alloc(tslot, kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t trow = tbase + ((uint32_t)(32 * quarter) << 16);

    // chunk 0's tiles and decay
    if (tid == 0) {
        mbar_arrive_tx(full_cb, kTxCB);
        mbar_arrive_tx(full_x, tx_x);
        for (int hb = 0; hb < 2; ++hb) {
            tma_2d(sC + hb * 16384, &m.C, 64 * hb, bc_row, full_cb);
            tma_2d(sB + hb * 16384, &m.B, 64 * hb, bc_row, full_cb);
            tma_2d(sX + hb * 8192, &m.u, 64 * hb, x_row, full_x);
            if (gate) tma_2d(sZ + hb * 8192, &m.z, 64 * hb, x_row, full_x);
        }
    }
    // warp 0: the decay vectors of chunk 0, and the delta bits of chunk 1 one chunk ahead
    uint2 dnext = make_uint2(0u, 0u);
    if (warp == 0) {
        chunk_decay(p, delta_bits(p, b, h, 0, lane), Ah, bias, lane, sdec, sdec + kQ, sdec + 2 * kQ);
        if (nchunks > 1) dnext = delta_bits(p, b, h, kQ, lane);
    }

    // the state: row n = row, channels p0 .. p0+15; skip weights of those channels
    float H[16], Dv[16];
    const bool have_h0 = p.h0 != nullptr;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int64_t d = d0 + p0 + k;
        H[k] = have_h0 ? __ldg(p.h0 + (b * Dm + d) * kN + row) : 0.f;
        Dv[k] = p.D ? __ldg(p.D + d) : 0.f;
    }
    if (have_h0) {
#pragma unroll
        for (int k = 0; k < 16; k += 8) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = H[k + e];
            store_pair8(sHhi, sHlo, row, p0 + k, v);
        }
        tc::fence_async_smem();
    }
    __syncthreads();

    bool failed = false;
    uint64_t* last_bar = nullptr;   // thread 0: the barrier of its latest commit and that phase
    unsigned last_ph = 0;
    int pend_cb = 0, pend_x = 0;    // thread 0: the chunk whose C, B (X, z) loads are in flight, or -1
    for (int c = 0; c < nchunks; ++c) {
        const int64_t t0 = (int64_t)c * kQ;
        const unsigned ph = (unsigned)c & 1u;
        const float* sdt = sdec + (c & 1) * kDec;
        const float* scum = sdt + kQ;
        const float* sw = sdt + 2 * kQ;
        const bool with_state = c > 0 || have_h0;

        // ---- G = C B^T once the chunk's C and B tiles are in (thread 0 waits for them and
        // issues; a wait that runs out is carried to the next CTA-wide vote)
        bool ok = true;
        if (tid == 0) {
            ok = mbar_wait(full_cb, ph, budget, p.status);
            if (ok) pend_cb = -1;
        }
        if (tid == 0 && ok) {
            tc::fence_after();
            constexpr uint32_t id = tc::idesc_bf16(128, 128, true, true);
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk)
                tc::mma_bf16(tbase + kColG, tc::desc(sC + kk * 2048, 16384, 1024, tc::kSwizzle128),
                             tc::desc(sB + kk * 2048, 16384, 1024, tc::kSwizzle128), id, kk > 0 ? 1u : 0u);
            tc::commit(mb_g);
            last_bar = mb_g;
            last_ph = ph;
        }
        // meanwhile: the next chunk's decay, and this step's gate inputs
        if (warp == 0 && c + 1 < nchunks) {
            float* nd = sdec + ((c + 1) & 1) * kDec;
            chunk_decay(p, dnext, Ah, bias, lane, nd, nd + kQ, nd + 2 * kQ);
            if (c + 2 < nchunks) dnext = delta_bits(p, b, h, t0 + 2 * kQ, lane);
        }

        // every thread waits for G itself
        ok = ok && mbar_wait(mb_g, ph, budget, p.status);
        tc::fence_after();

        // ---- M = G o decay mask: row i = row, steps j0 .. j0+31 (a warp whose steps all lie
        // after its rows writes zeros: the causal mask)
        if (!ok) {
            // a wait ran out: nothing to build, the vote below ends the loop
        } else if (j0 > (uint32_t)(32 * quarter + 31)) {
            const float zero8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 32; k += 8)
                store_pair8(sMhi + (j0 >> 6) * 16384, sMlo + (j0 >> 6) * 16384, row, (j0 & 63u) + k, zero8);
        } else {
            uint32_t gv[32];
            tc::ld32(trow + kColG + j0, gv);
            const float ci = scum[row];
            tc::wait_ld();
            tc::after_wait(gv);
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
                float cj[8], dj[8];
                lds8f(scum + j0 + k, cj);
                lds8f(sdt + j0 + k, dj);
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = j0 + k + e;
                    v[e] = j <= row ? __uint_as_float(gv[k + e]) * ex2_approx(ci - cj[e]) * dj[e] : 0.f;
                }
                store_pair8(sMhi + (j0 >> 6) * 16384, sMlo + (j0 >> 6) * 16384, row, (j0 & 63u) + k, v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
        ok = ok && mbar_wait(full_x, ph, budget, p.status);
        if (tid == 0 && ok) pend_x = -1;
        if (__syncthreads_or(!ok)) { failed = true; break; }

        // ---- Y = M X (K-major, K = j) and C H (MN-major, K = n)
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
        // every thread waits for Y and C H itself
        ok = mbar_wait(mb_y, ph, budget, p.status);
        tc::fence_after();

        // ---- outputs of step i = row, channels p0 .. p0+15
        if (ok) {
            uint32_t yv[16], cv[16];
            tc::ld16(trow + kColY + p0, yv);
            if (with_state) tc::ld16(trow + kColCH + p0, cv);
            tc::wait_ld();
            tc::after_wait(yv);
            if (with_state) tc::after_wait(cv);
            const float e = with_state ? ex2_approx(scum[row]) : 0.f;
            const unsigned char* xt = sX + (row >> 6) * 8192;
            unsigned char* zt = sZ + (row >> 6) * 8192;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float x = bf16_at(xt, p0 + k, row & 63u);
                float v = __uint_as_float(yv[k]);
                if (with_state) v = fmaf(e, __uint_as_float(cv[k]), v);
                v = fmaf(Dv[k], x, v);
                unsigned short* slot = reinterpret_cast<unsigned short*>(zt + tc::sw128_off(p0 + k, row & 63u));
                if (gate) v *= silu1(__bfloat162float(__ushort_as_bfloat16(*slot)));
                *slot = __bfloat16_as_ushort(__float2bfloat16_rn(v));   // out(p, t) where z(p, t) was
            }
        }
        // ---- X' = diag(w) X as hi + lo in the M tile (free once Y is done): two 8-step
        // pieces of a head-dim row per thread, laid out like the X tile (K-major, K = step)
        if (ok) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t e = (uint32_t)tid + (uint32_t)r * kThreadsSsd;   // 0 .. 1023
                const uint32_t pp = e >> 4, s8 = (e & 15u) * 8u;                  // head-dim row, first step
                const uint4 raw = *reinterpret_cast<const uint4*>(sX + (s8 >> 6) * 8192 + tc::sw128_off(pp, s8 & 63u));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                float wj[8], v[8];
                lds8f(sw + s8, wj);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t bits = (k & 1) ? (w4[k >> 1] & 0xFFFF0000u) : (w4[k >> 1] << 16);
                    v[k] = __uint_as_float(bits) * wj[k];
                }
                store_pair8(sMhi + (s8 >> 6) * 8192, sMlo + (s8 >> 6) * 8192, pp, s8 & 63u, v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
        if (__syncthreads_or(!ok)) { failed = true; break; }

        // ---- the out tile (written over the z tile) to global; S = B^T X' (B, K-major, straight
        // from its TMA tile); then the next chunk's C tile (B is read until S is done)
        if (tid == 0) {
            tma_store_2d(&m.out, (int)t0, x_row, sZ);
            tma_store_2d(&m.out, (int)t0 + 64, x_row, sZ + 8192);
            bulk_commit();
            tc::fence_after();
            constexpr uint32_t ids = tc::idesc_bf16(128, kP, false, false);
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk) {
                const uint64_t ab = tc::desc(sB + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, tc::kSwizzle128);
                const int xo = (kk >> 2) * 8192 + (kk & 3) * 32;
                tc::mma_bf16(tbase + kColS, ab, tc::desc(sMhi + xo, 16, 1024, tc::kSwizzle128), ids, kk > 0 ? 1u : 0u);
                tc::mma_bf16(tbase + kColS, ab, tc::desc(sMlo + xo, 16, 1024, tc::kSwizzle128), ids, 1u);
            }
            tc::commit(mb_s);
            last_bar = mb_s;
            last_ph = ph;
            if (c + 1 < nchunks) {
                pend_cb = c + 1;
                mbar_arrive_tx(full_cb, kTxCB);   // C now, B once S has read it
                for (int hb = 0; hb < 2; ++hb) tma_2d(sC + hb * 16384, &m.C, (int)(t0 + kQ + 64 * hb), bc_row, full_cb);
            }
        }
        // every thread waits for S itself
        ok = mbar_wait(mb_s, ph, budget, p.status);
        tc::fence_after();
        // the next chunk's X and z tiles (this chunk's MMAs that read X are complete, and
        // its outputs were written before the barrier above)
        // the out tile must be read out of shared memory before the z tile is loaded over it,
        // or (no gate) before the next chunk's outputs are written there after the barriers below
        if (tid == 0) bulk_wait_read();
        if (tid == 0 && ok && c + 1 < nchunks) {
            for (int hb = 0; hb < 2; ++hb) tma_2d(sB + hb * 16384, &m.B, (int)(t0 + kQ + 64 * hb), bc_row, full_cb);
            pend_x = c + 1;
            mbar_arrive_tx(full_x, tx_x);
            for (int hb = 0; hb < 2; ++hb) {
                tma_2d(sX + hb * 8192, &m.u, (int)(t0 + kQ + 64 * hb), x_row, full_x);
                if (gate) tma_2d(sZ + hb * 8192, &m.z, (int)(t0 + kQ + 64 * hb), x_row, full_x);
            }
        }

        // ---- H = 2^cum_end H + S (row n = row, channels p0 .. p0+15)
        if (ok) {
            uint32_t sv[16];
            tc::ld16(trow + kColS + p0, sv);
            tc::wait_ld();
            tc::after_wait(sv);
            const float dec = ex2_approx(scum[kQ - 1]);
#pragma unroll
            for (int k = 0; k < 16; ++k) H[k] = fmaf(dec, H[k], __uint_as_float(sv[k]));
#pragma unroll
            for (int k = 0; k < 16; k += 8) {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = H[k + e];
                store_pair8(sHhi, sHlo, row, p0 + k, v);
            }
        }
        tc::fence_async_smem();
        tc::fence_before();
        if (__syncthreads_or(!ok)) { failed = true; break; }   // H tile and the next chunk's decay are visible
    }
    if (!failed && p.last_state) {
#pragma unroll
        for (int k = 0; k < 16; ++k) p.last_state[(b * Dm + d0 + p0 + k) * kN + row] = H[k];
    }
    // release TMEM and shared memory once nothing can still write them: after a failed wait,
    // wait (bounded) for the last tensor-core batch this CTA committed and its loads in flight
    if (failed && tid == 0) {
        if (last_bar) mbar_wait(last_bar, last_ph, budget, p.status);
        if (pend_cb >= 0) mbar_wait(full_cb, (unsigned)pend_cb & 1u, budget, p.status);
        if (pend_x >= 0) mbar_wait(full_x, (unsigned)pend_x & 1u, budget, p.status);
    }
    if (tid == 0) bulk_wait_all();   // the last out tile is written before shared memory goes away
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
    // every launch: the attribute belongs to the current device's instance of the kernel
    if (cudaFuncSetAttribute(ssd_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemSsd) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (grid <= 0) return SSM_OK;
    ssd_fwd_kernel<<<(unsigned)grid, kThreadsSsd, kSmemSsd, s>>>(prm, maps);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace ssm
