// Backward of the selective scan: the gradients of every input of the forward
// scan, given dout (and optionally the gradient of the final state).  The
// states are not stored by the forward; this pass recomputes them ("Agent
// 229: SSM optimization patterns" page, section 4 "Activation Recomputation",
// checkpoints at chunk boundaries; Mamba "architecture-details" page, "Memory
// Efficiency": training recomputes activations in the backward pass).
// Declared in include/ssm_scan.h as ssm_selective_scan_bwd.
//
// With x_t = delta_t + bias, dt_t = softplus(x_t), dA_tn = exp(dt_t a_n),
// h_t = dA_t h_(t-1) + dt_t B_t u_t, y_t = C_t.h_t + D u_t, out_t = y_t silu(z_t)
// and g the gradient of the state carried from t+1 (g = dlast after the last
// step), walking t down:
//
//   dy = dout silu(z)             g_n += dy C_tn   (dLoss/dh_tn)
//   dB_tn += g_n dt u_t           dC_tn += dy h_tn           (summed over channels)
//   du_t = dt sum_n g_n B_tn + dy D
//   ddt_t = u_t sum_n g_n B_tn + sum_n g_n h_(t-1)n a_n dA_tn
//   da_n += g_n h_(t-1)n dt dA_tn,   then g_n <- dA_tn g_n (carried to t-1)
//   ddelta_t = ddt_t sigmoid(x_t),  dbias += ddelta_t,  dz_t = dout y_t silu'(z_t)
//
// A tile is 32 channels of one batch row (S6 layout, dstate 16), run by eight
// warps, each four channels x 8 lanes x 2 states.  Its sequence is cut into
// segments, and the work units (tile, segment) go to persistent CTAs from a
// ticket counter: first every forward unit, segment-major, then every reverse
// unit, last segment first.  A forward unit runs the recurrence from the state
// its predecessor handed over and stores the state at the start of every 32-step
// block (the checkpoints).  A reverse unit takes the state gradient from the
// segment after it and walks its blocks backwards: per block it runs the
// recurrence forward from the block's checkpoint to get the states at the four
// 8-step window starts (shared memory), then per window recomputes the 8 states and
// decays into registers and runs the window in reverse.  Given the forward's stored
// states (one per 8-step window, ssm_selective_scan_bwd_ckpt), no forward unit runs and
// the window starts are copied in with the block's rows instead of rebuilt.  A unit waits (bounded) only on units with smaller
// tickets, which running CTAs hold, so the chain always progresses.  Each block's
// 32-step rows of the inputs are staged in shared memory by cp.async, double
// buffered: a block's prologue issues the next block's rows.
//
// Sums over the states (y, sum g B, the decay term) are transposed shuffle
// reductions inside the 8 lanes of a channel.  dB and dC, sums over channels, are
// summed over a warp's four channels by shuffles at every step, then over the
// eight warps through shared memory once per 32-step block, and the tile's sums
// are added into dB and dC by vector atomic adds (red.global.add.v4.f32) that
// resolve in L2: no per-tile rows reach HBM, and the order of the adds between
// tiles, so the last bits of dB and dC, may differ between calls.  A second
// kernel adds the per-row dA, dD and dbias partials in a fixed order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "bwd_generic.h"
#include "scan_kernel.cuh"   // ex2_approx, rcp_approx, softplus1, kLog2e
#include "ssm_scan.h"

namespace ssm {
namespace {

constexpr int kN = 16;         // states per channel
constexpr int kBT = 32;        // steps per staged block
constexpr int kWin = 8;        // steps per recomputed window (= one 8-lane reduction)
// A CTA of NW warps (8, or 4 where 32-channel tiles would leave CTA slots idle), each
// warp 4 channels x 8 lanes x 2 states.
template <int NW>
struct Bw {
    static constexpr int CT = 4 * NW;                   // channels per CTA (a tile)
    static constexpr int THREADS = 32 * NW;
    static constexpr int STAGE_ROWS = 4 * CT + 2 * kN;  // u, delta, z, dout rows; B, C rows
};

struct BwdParams {
    const void *u, *delta, *z, *dout, *B, *C;
    const float *A, *D, *bias, *h0, *dlast;
    void *du, *ddelta, *dz;
    float* dh0;
    // workspace
    unsigned* ticket;            // work-unit counter (zeroed before the launch)
    int* status;                 // kernel-side ssm_status_t
    unsigned *flag1, *flag2;     // [tile][seg]: forward / reverse segment done (zeroed before the launch)
    float *carry1, *carry2;      // [tile][seg][CT][kN]: state after / state gradient before a segment
    // the kernel's checkpoints [b * dim + d][block][kN] (the state entering each 32-step block),
    // or with ext_ckpt the forward's stored states [b * dim + d][window][kN] (the state entering
    // each 8-step window); then no forward units run
    float* ckpt;
    int ext_ckpt;
    float *dB, *dC;              // the outputs (batch, groups, kN, L), zeroed before the launch
    int red_vec;                 // 16-byte atomic adds into dB, dC (L % 4 == 0, aligned bases)
    float *dAp, *dDp, *dbp;      // per segment and (b, d) row: [seg][row][kN], [seg][row], [seg][row]
    int64_t batch, dim, seqlen, ngroups;
    int64_t ntiles;              // batch * dim / CT (channels per tile)
    int tiles_per_row;           // dim / CT
    int nseg, seg_blocks;        // segments per tile, 32-step blocks per segment
    int softplus;
    uint64_t budget_ns;          // bounded waits
    unsigned need;               // the flag value a wait waits for: 1, or 2 (never written) under the test hook
};

template <typename T> struct Io;
template <> struct Io<float> {
    using raw = float;
    __device__ static float f(raw v) { return v; }
    __device__ static raw from(float v) { return v; }
};
template <> struct Io<__nv_bfloat16> {
    using raw = unsigned short;
    __device__ static float f(raw v) { return __uint_as_float((uint32_t)v << 16); }
    __device__ static raw from(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
};

// shared memory (bytes).  The per-step rows P and U have kPS = kBT + 1 entries per
// channel, so the four channels a warp reads at one step sit in different banks.
constexpr int kPS = kBT + 1;
template <typename T, int NW>
struct Smem {
    static constexpr int CT = Bw<NW>::CT;
    static constexpr int kRow = kBT * (int)sizeof(T) + 16;        // staged row stride (16-byte padded)
    static constexpr int STAGE = 0;                               // two buffers of staged rows
    // in each stage buffer after the rows: the states entering the block's four windows,
    // float [CT][kWinStride] (a channel's 4 x kN, padded so that two channels' reads of one
    // window meet different banks)
    static constexpr int kWinStride = (kBT / kWin) * kN + 16;
    static constexpr int WINS = Bw<NW>::STAGE_ROWS * kRow;
    static constexpr int kStageBytes = WINS + CT * kWinStride * 4;
    // Per-step values in 8-byte pairs: a lane reads only the pairs a pass needs (the
    // shared-memory pipe moves a lane's bytes, broadcast or not).
    static constexpr int PA = STAGE + 2 * kStageBytes;            // float2 [CT][kPS]: dt, dt*u
    static constexpr int PB = PA + CT * kPS * 8;                  // float2 [CT][kPS]: dy, dout*silu'(z)
    static constexpr int U = PB + CT * kPS * 8;                   // float2 [CT][kPS]: u, sigmoid(x)
    static constexpr int BS = U + CT * kPS * 8;                   // float2 [kBT][8]: B_2j, B_2j+1
    static constexpr int CS = BS + kBT * 8 * 8;                   // float2 [kBT][8]: C_2j, C_2j+1
    // per window and warp, the dB, dC terms summed over the warp's channels:
    // float [kBT/kWin windows][NW warps][4 components][8 lanes j][kWin steps]
    static constexpr int RED = CS + kBT * 8 * 8;
    static constexpr int TOTAL = RED + (kBT / kWin) * NW * 4 * 8 * kWin * 4;
};

// rows x kBT steps [t0, t0 + kBT) of `rows` rows (row r at src + r * stride) into
// shared memory, zero past L.  vec: asynchronous 16-byte copies (rows 16-byte
// aligned, L a multiple of the chunk; complete after cp_async_wait), else element by
// element.
template <typename T, int NW>
__device__ __forceinline__ void stage_rows(unsigned char* dst, const T* src, int64_t stride, int rows, int64_t t0,
                                           int64_t L, bool vec, int tid) {
    constexpr int kThreads = Bw<NW>::THREADS;
    using R = typename Io<T>::raw;
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int CPR = kBT / E;
    if (vec) {
        // cp.async: zero-filled when the chunk lies past L (then the source is not read)
        for (int i = tid; i < rows * CPR; i += kThreads) {
            const int r = i / CPR, k = i % CPR;
            const int64_t t = t0 + (int64_t)k * E;
            const T* g = src + r * stride + (t < L ? t : 0);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst + r * Smem<T, NW>::kRow + k * 16)),
                         "l"(g), "r"(t < L ? 16 : 0)
                         : "memory");
        }
    } else {
        const R* s = reinterpret_cast<const R*>(src);
        for (int i = tid; i < rows * kBT; i += kThreads) {
            const int r = i / kBT, k = i % kBT;
            const int64_t t = t0 + k;
            reinterpret_cast<R*>(dst + r * Smem<T, NW>::kRow)[k] = t < L ? s[r * stride + t] : (R)0;
        }
    }
}

__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The forward's stored states entering windows [win0, win0 + 4) of the tile's CT channels
// (channel cc's row at ck + cc * nwin * kN) into the block's window area, zero past nwin.
// vec: 16-byte asynchronous copies (ck 16-byte aligned), else element by element.
template <typename T, int NW>
__device__ __forceinline__ void stage_wins(float* dst, const float* ck, int64_t nwin, int64_t win0, bool vec,
                                           int tid) {
    constexpr int kCT = Bw<NW>::CT, kThreads = Bw<NW>::THREADS;
    constexpr int CPC = (kBT / kWin) * kN / 4;   // 16-byte chunks per channel
    for (int i = tid; i < kCT * CPC; i += kThreads) {
        const int cc = i / CPC, k = i % CPC;
        const int64_t win = win0 + k / (kN / 4);
        const bool in = win < nwin;
        const float* g = ck + ((int64_t)cc * nwin + (in ? win : 0)) * kN + (k % (kN / 4)) * 4;
        float* sm = dst + cc * Smem<T, NW>::kWinStride + k * 4;
        if (vec) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sm)), "l"(g), "r"(in ? 16 : 0)
                         : "memory");
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) sm[e] = in ? g[e] : 0.f;
        }
    }
}

template <typename T>
__device__ __forceinline__ float staged(const unsigned char* base, int row, int k) {
    return Io<T>::f(reinterpret_cast<const typename Io<T>::raw*>(base + row * Smem<T, 8>::kRow)[k]);
}

// a (B_2j, B_2j+1) or (C_2j, C_2j+1) pair in shared memory: two bf16 in one word for bf16
// I/O (half the shared-memory bytes; unpacked on use), a float2 for fp32
template <typename T> struct BCPair;
template <> struct BCPair<float> {
    using W = float2;
    __device__ static W pack(float a, float b) { return make_float2(a, b); }
    __device__ static float2 get(W w) { return w; }
};
template <> struct BCPair<__nv_bfloat16> {
    using W = uint32_t;
    __device__ static W pack(float a, float b) {
        return (__float_as_uint(b) & 0xFFFF0000u) | (__float_as_uint(a) >> 16);   // exact: a, b are bf16 values
    }
    __device__ static float2 get(W w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)); }
};

__device__ __forceinline__ float sigmoid1(float x) { return rcp_approx(1.f + ex2_approx(x * -kLog2e)); }

// One step of the recurrence on the lane's two states, as f32x2 pairs (the same
// expression in both passes, so the recomputed states equal the checkpointed ones
// bit for bit).
__device__ __forceinline__ void fwd_step(float2& h, float2& dA, float dt, float dtu, float b0, float b1, float2 al) {
    const float2 arg = mul2(dup2(dt), al);
    dA = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
    h = fma2(dA, h, mul2(dup2(dtu), make_float2(b0, b1)));
}

// Sum of v over the 8 lanes of a channel (lane bits 0-2 = j), transposed: lane j
// gets the total of element j.  Three halvings, 4 + 2 + 1 shuffles.
__device__ __forceinline__ float reduce8(const float (&v)[8], int j) {
    float a[4], b[2];
    const bool h2 = j & 4, h1 = j & 2, h0 = j & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = h2 ? v[i] : v[i + 4];
        const float keep = h2 ? v[i + 4] : v[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = h1 ? a[i] : a[i + 2];
        const float keep = h1 ? a[i + 2] : a[i];
        b[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const float send = h0 ? b[0] : b[1];
    const float keep = h0 ? b[1] : b[0];
    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

__device__ __forceinline__ void red_add_v4(float* dst, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// The dB, dC terms of one 32-step block, held per (window, warp) in shared memory,
// summed over the NW warps in a fixed order and added into dB and dC (rows of the
// tile's group, dBg / dCg) by atomic adds: each of the 256 items is four consecutive
// steps of one (window, component, lane j).
template <int NW>
__device__ __forceinline__ void red_add(const float* red, float* dBg, float* dCg, int64_t t0, int64_t L, bool vec,
                                       int tid) {
#pragma unroll
    for (int it = tid; it < 256; it += Bw<NW>::THREADS) {
        const int w = it >> 6, comp = (it >> 4) & 3, jj = (it >> 1) & 7, q4 = (it & 1) * 4;
        const int within = comp * 64 + jj * 8 + q4;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int wp = 0; wp < NW; ++wp) {
            const float4 v = *reinterpret_cast<const float4*>(red + (w * NW + wp) * 256 + within);
            s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
        }
        const int64_t ta = t0 + w * kWin + q4;
        float* dst = ((comp & 2) ? dCg : dBg) + (int64_t)(2 * jj + (comp & 1)) * L + ta;
        if (vec && ta + 3 < L) {
            red_add_v4(dst, s);
        } else {
            const float e[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (ta + i < L) atomicAdd(dst + i, e[i]);
        }
    }
}

template <typename T, int NW>
__global__ void __launch_bounds__(32 * NW, 16 / NW) scan_bwd_kernel(const BwdParams p) {
    using S = Smem<T, NW>;
    constexpr int kCT = Bw<NW>::CT, kThreads = Bw<NW>::THREADS;
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char* stage_base = smem + S::STAGE;
    float2* sPa = reinterpret_cast<float2*>(smem + S::PA);
    float2* sPb = reinterpret_cast<float2*>(smem + S::PB);
    float2* sU = reinterpret_cast<float2*>(smem + S::U);
    using BW = BCPair<T>;
    typename BW::W* sB = reinterpret_cast<typename BW::W*>(smem + S::BS);
    typename BW::W* sC = reinterpret_cast<typename BW::W*>(smem + S::CS);
    float* sR = reinterpret_cast<float*>(smem + S::RED);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = lane >> 3, j = lane & 7;
    const int c = warp * 4 + q;                    // channel within the tile
    __shared__ unsigned s_ticket;
    const int64_t L = p.seqlen, Dm = p.dim, G = p.ngroups;
    const int64_t rows = p.batch * Dm;
    const bool vec = (L % (16 / (int64_t)sizeof(T))) == 0 &&
                     ((reinterpret_cast<uintptr_t>(p.u) | reinterpret_cast<uintptr_t>(p.delta) |
                       reinterpret_cast<uintptr_t>(p.z) | reinterpret_cast<uintptr_t>(p.dout) |
                       reinterpret_cast<uintptr_t>(p.B) | reinterpret_cast<uintptr_t>(p.C)) & 15u) == 0;
    const int nblk = (int)((L + kBT - 1) / kBT);
    const int64_t per_pass = p.ntiles * p.nseg;
    const int64_t nfwd = p.ext_ckpt ? 0 : per_pass;   // forward units come first, when they run

    for (;;) {
        __syncthreads();   // the previous unit is done with shared memory and s_ticket
        if (tid == 0) s_ticket = atomicAdd(p.ticket, 1u);
        __syncthreads();
        const int64_t k = s_ticket;
        if (k >= nfwd + per_pass) break;
        const bool fwd = k < nfwd;
        const int64_t kk = fwd ? k : k - nfwd;
        const int seg = fwd ? (int)(kk / p.ntiles) : p.nseg - 1 - (int)(kk / p.ntiles);
        const int64_t tile = kk % p.ntiles;        // = b * tiles_per_row + tile in the row
        const int64_t b = tile / p.tiles_per_row;
        const int64_t row0 = tile * kCT;           // first (b, d) row of the tile
        const int64_t d0 = row0 - b * Dm;
        const int64_t g = d0 / (Dm / G);
        const int64_t d = d0 + c;
        const T* u = static_cast<const T*>(p.u) + row0 * L;
        const T* dl = static_cast<const T*>(p.delta) + row0 * L;
        const T* zz = p.z ? static_cast<const T*>(p.z) + row0 * L : nullptr;
        const T* go = static_cast<const T*>(p.dout) + row0 * L;
        const T* Bg = static_cast<const T*>(p.B) + (b * G + g) * kN * L;
        const T* Cg = static_cast<const T*>(p.C) + (b * G + g) * kN * L;
        float* ckpt = p.ckpt + (row0 + c) * (int64_t)nblk * kN + 2 * j;   // this thread's states, block 0
        const int blk0 = seg * p.seg_blocks;
        const int blk1 = min(nblk, blk0 + p.seg_blocks);
        const int64_t us = tile * p.nseg + seg;    // this unit's flag / carry slot
        const float2 Aln = make_float2(__ldg(p.A + d * kN + 2 * j), __ldg(p.A + d * kN + 2 * j + 1));
        const float2 al = make_float2(Aln.x * kLog2e, Aln.y * kLog2e);
        const float Dc = p.D ? __ldg(p.D + d) : 0.f;

        // bounded waits (thread 0) for the units this one depends on; a wait that runs out, or
        // a status already set by another CTA, records the failure and the unit goes on with
        // whatever it finds (the call then reports SSM_ERR_TIMEOUT and its outputs are invalid)
        if (tid == 0) {
            bool ok = true;
            const unsigned* need[2] = {nullptr, nullptr};
            if (fwd && seg > 0) need[0] = p.flag1 + us - 1;
            if (!fwd) {
                if (!p.ext_ckpt) need[0] = p.flag1 + us;
                if (seg + 1 < p.nseg) need[1] = p.flag2 + us + 1;
            }
            for (int w = 0; w < 2; ++w) {
                if (!need[w]) continue;
                const uint64_t t_start = now_ns();
                while (ld_acquire(need[w]) < p.need) {
                    __nanosleep(128);   // leave the issue slots to the working warps of this SM
                    if (*reinterpret_cast<volatile int*>(p.status) != SSM_OK) { ok = false; break; }
                    if (now_ns() - t_start > p.budget_ns) {
                        atomicCAS(p.status, SSM_OK, SSM_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
            }
        }
        __syncthreads();

        if (fwd) {
            // ---------------- forward unit: the recurrence, checkpoints at every block start
            float2 h;
            if (seg == 0)
                h = p.h0 ? *reinterpret_cast<const float2*>(p.h0 + (row0 + c) * kN + 2 * j) : make_float2(0.f, 0.f);
            else
                h = __ldcg(reinterpret_cast<const float2*>(p.carry1 + ((us - 1) * kCT + c) * kN + 2 * j));
            // the rows of the unit's first block; each block's prologue then issues the next's
            auto issue_fwd = [&](unsigned char* sg, int64_t ts) {
                stage_rows<T, NW>(sg, u, L, kCT, ts, L, vec, tid);
                stage_rows<T, NW>(sg + kCT * S::kRow, dl, L, kCT, ts, L, vec, tid);
                stage_rows<T, NW>(sg + 4 * kCT * S::kRow, Bg, L, kN, ts, L, vec, tid);
            };
            issue_fwd(stage_base, (int64_t)blk0 * kBT);
            int cur = 0;
            for (int blk = blk0; blk < blk1; ++blk, cur ^= 1) {
                const int64_t t0 = (int64_t)blk * kBT;
                unsigned char* stage = stage_base + cur * S::kStageBytes;
                cp_async_wait();
                __syncthreads();   // this block's rows are in; the previous block is done with P and BC
                // dt and dt*u of this warp's 4 channels, lane = step
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int cc = warp * 4 + i;
                    const float uv = staged<T>(stage, cc, lane);
                    const float xv =
                        staged<T>(stage + kCT * S::kRow, cc, lane) + (p.bias ? __ldg(p.bias + d0 + cc) : 0.f);
                    float dt = p.softplus ? softplus1(xv) : xv;
                    if (t0 + lane >= L) dt = 0.f;
                    sPa[cc * kPS + lane] = make_float2(dt, dt * uv);
                }
                for (int it = tid; it < kBT * 8; it += kThreads) {
                    const int t = it >> 3, jj = it & 7;
                    const unsigned char* sb = stage + 4 * kCT * S::kRow;
                    sB[t * 8 + jj] = BW::pack(staged<T>(sb, 2 * jj, t), staged<T>(sb, 2 * jj + 1, t));
                }
                // the next block's rows go into the other buffer, read last by the previous block
                if (blk + 1 < blk1) issue_fwd(stage_base + (cur ^ 1) * S::kStageBytes, t0 + kBT);
                __syncthreads();
                *reinterpret_cast<float2*>(ckpt + (int64_t)blk * kN) = h;
#pragma unroll
                for (int w = 0; w < kBT / kWin; ++w) {
#pragma unroll 4
                    for (int t = w * kWin; t < (w + 1) * kWin; ++t) {
                        const float2 pv = sPa[c * kPS + t];
                        const float2 bb = BW::get(sB[t * 8 + j]);
                        float2 dA;
                        fwd_step(h, dA, pv.x, pv.y, bb.x, bb.y, al);
                    }
                }
            }
            // hand the state to the next segment; the checkpoints go with it
            *reinterpret_cast<float2*>(p.carry1 + (us * kCT + c) * kN + 2 * j) = h;
            __syncthreads();
            if (tid == 0) {
                __threadfence();
                st_release(p.flag1 + us, 1u);
            }
            continue;
        }

        // ---------------- reverse unit: blocks backwards, windows recomputed from the block checkpoints
        float2 gs;
        if (seg + 1 < p.nseg)
            gs = __ldcg(reinterpret_cast<const float2*>(p.carry2 + ((us + 1) * kCT + c) * kN + 2 * j));
        else
            gs = p.dlast ? *reinterpret_cast<const float2*>(p.dlast + (row0 + c) * kN + 2 * j) : make_float2(0.f, 0.f);
        float2 dAacc = make_float2(0.f, 0.f);
        float dbias = 0.f, dDacc = 0.f;
        float* dBg = p.dB + (b * G + g) * kN * L;
        float* dCg = p.dC + (b * G + g) * kN * L;
        const bool rvec = p.red_vec != 0;
        // the checkpoint of the block being walked (the next, earlier one is fetched a block
        // ahead); with the forward's states, the window starts come with the block's rows
        const bool ext = p.ext_ckpt != 0;
        float2 hblk = ext ? make_float2(0.f, 0.f)
                          : __ldcg(reinterpret_cast<const float2*>(ckpt + (int64_t)(blk1 - 1) * kN));
        const int64_t nwin = (L + kWin - 1) / kWin;
        const float* cktile = p.ckpt + row0 * nwin * kN;
        const bool ckvec = (reinterpret_cast<uintptr_t>(p.ckpt) & 15u) == 0;
        auto issue_rev = [&](unsigned char* sg, int64_t ts) {
            if (ext) stage_wins<T, NW>(reinterpret_cast<float*>(sg + S::WINS), cktile, nwin, ts / kWin, ckvec, tid);
            stage_rows<T, NW>(sg, u, L, kCT, ts, L, vec, tid);
            stage_rows<T, NW>(sg + kCT * S::kRow, dl, L, kCT, ts, L, vec, tid);
            if (zz) stage_rows<T, NW>(sg + 2 * kCT * S::kRow, zz, L, kCT, ts, L, vec, tid);
            stage_rows<T, NW>(sg + 3 * kCT * S::kRow, go, L, kCT, ts, L, vec, tid);
            stage_rows<T, NW>(sg + 4 * kCT * S::kRow, Bg, L, kN, ts, L, vec, tid);
            stage_rows<T, NW>(sg + (4 * kCT + kN) * S::kRow, Cg, L, kN, ts, L, vec, tid);
        };
        issue_rev(stage_base, (int64_t)(blk1 - 1) * kBT);
        int cur = 0;
        for (int blk = blk1 - 1; blk >= blk0; --blk, cur ^= 1) {
            const int64_t t0 = (int64_t)blk * kBT;
            unsigned char* stage = stage_base + cur * S::kStageBytes;
            cp_async_wait();
            __syncthreads();   // this block's rows are in; the previous block is done with P, U, BC
            // the previous block's dB, dC terms (every warp has written them)
            if (blk + 1 < blk1) red_add<NW>(sR, dBg, dCg, t0 + kBT, L, rvec, tid);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cc = warp * 4 + i;
                const bool valid = t0 + lane < L;
                const float uv = staged<T>(stage, cc, lane);
                const float xv =
                    staged<T>(stage + kCT * S::kRow, cc, lane) + (p.bias ? __ldg(p.bias + d0 + cc) : 0.f);
                const float gov = staged<T>(stage + 3 * kCT * S::kRow, cc, lane);
                float dt = p.softplus ? softplus1(xv) : xv;
                float sp = p.softplus ? sigmoid1(xv) : 1.f;
                if (!valid) dt = sp = 0.f;
                float dy = gov, dzf = 0.f;
                if (zz) {
                    const float zv = staged<T>(stage + 2 * kCT * S::kRow, cc, lane);
                    const float sg = sigmoid1(zv);
                    dy = gov * zv * sg;
                    dzf = gov * (sg * fmaf(zv, 1.f - sg, 1.f));
                }
                sPa[cc * kPS + lane] = make_float2(dt, dt * uv);
                sPb[cc * kPS + lane] = make_float2(dy, dzf);
                sU[cc * kPS + lane] = make_float2(uv, sp);
            }
            for (int it = tid; it < kBT * 8; it += kThreads) {
                const int t = it >> 3, jj = it & 7;
                const unsigned char* sb = stage + 4 * kCT * S::kRow;
                const unsigned char* sc = stage + (4 * kCT + kN) * S::kRow;
                sB[t * 8 + jj] = BW::pack(staged<T>(sb, 2 * jj, t), staged<T>(sb, 2 * jj + 1, t));
                sC[t * 8 + jj] = BW::pack(staged<T>(sc, 2 * jj, t), staged<T>(sc, 2 * jj + 1, t));
            }
            // the next (earlier) block's rows go into the other buffer
            if (blk > blk0) issue_rev(stage_base + (cur ^ 1) * S::kStageBytes, t0 - kBT);
            __syncthreads();

            // the states entering the four windows: staged with the rows (the forward's), or by
            // the recurrence from the block checkpoint
            float* wins = reinterpret_cast<float*>(stage + S::WINS) + c * S::kWinStride + 2 * j;
            if (!ext) {
                const float2 hprev =
                    blk > blk0 ? __ldcg(reinterpret_cast<const float2*>(ckpt + (int64_t)(blk - 1) * kN))
                               : make_float2(0.f, 0.f);
                float2 hh = hblk;
#pragma unroll
                for (int w = 0; w < kBT / kWin; ++w) {
                    *reinterpret_cast<float2*>(wins + w * kN) = hh;
                    if (w + 1 < kBT / kWin) {
#pragma unroll 4
                        for (int t = w * kWin; t < (w + 1) * kWin; ++t) {
                            const float2 pv = sPa[c * kPS + t];
                            const float2 bb = BW::get(sB[t * 8 + j]);
                            float2 dA;
                            fwd_step(hh, dA, pv.x, pv.y, bb.x, bb.y, al);
                        }
                    }
                }
                hblk = hprev;
            }
            for (int w = kBT / kWin - 1; w >= 0; --w) {
                const int tw = w * kWin;   // first step of the window within the block
                const float2 he = *reinterpret_cast<const float2*>(wins + w * kN);   // the state entering the window
                float2 hr[kWin], dAr[kWin];
                float yw;   // y of step j of the window, summed over the states
                {
                    float2 hh = he;
                    float yp[kWin];
#pragma unroll
                    for (int t = 0; t < kWin; ++t) {
                        const float2 pv = sPa[c * kPS + tw + t];
                        const float2 bb = BW::get(sB[(tw + t) * 8 + j]);
                        const float2 cc = BW::get(sC[(tw + t) * 8 + j]);
                        fwd_step(hh, dAr[t], pv.x, pv.y, bb.x, bb.y, al);
                        hr[t] = hh;
                        yp[t] = fmaf(cc.x, hh.x, cc.y * hh.y);
                    }
                    yw = reduce8(yp, j);
                }
                float gb[kWin], qq[kWin], rw[kWin];
                const bool q1 = q & 2, q0 = q & 1;
#pragma unroll
                for (int t = kWin - 1; t >= 0; --t) {
                    const float2 pv = sPa[c * kPS + tw + t];   // dt, dt*u
                    const float dy = sPb[c * kPS + tw + t].x;
                    const float2 bb = BW::get(sB[(tw + t) * 8 + j]);
                    const float2 cc = BW::get(sC[(tw + t) * 8 + j]);
                    gs = fma2(dup2(dy), cc, gs);   // + dy C: now dLoss/dh_t
                    const float2 hp = t > 0 ? hr[t - 1] : he;
                    const float2 e = mul2(mul2(gs, hp), dAr[t]);
                    dAacc = fma2(e, dup2(pv.x), dAacc);
                    gb[t] = fmaf(gs.x, bb.x, gs.y * bb.y);
                    qq[t] = fmaf(e.x, Aln.x, e.y * Aln.y);
                    const float2 db = mul2(gs, dup2(pv.y)), dc = mul2(dup2(dy), hr[t]);
                    // the four terms (dB_2j, dB_2j+1, dC_2j, dC_2j+1) summed over the warp's four
                    // channels, transposed: lane (q, j) keeps component q
                    const float a0 = (q1 ? dc.x : db.x) + __shfl_xor_sync(0xffffffffu, q1 ? db.x : dc.x, 16);
                    const float a1 = (q1 ? dc.y : db.y) + __shfl_xor_sync(0xffffffffu, q1 ? db.y : dc.y, 16);
                    rw[t] = (q0 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, q0 ? a0 : a1, 8);
                    gs = mul2(gs, dAr[t]);           // carry to t-1
                }
                const float GB = reduce8(gb, j), Q = reduce8(qq, j);
                {
                    float4* rd = reinterpret_cast<float4*>(sR + ((w * NW + warp) * 4 + q) * 64 + j * 8);
                    rd[0] = make_float4(rw[0], rw[1], rw[2], rw[3]);
                    rd[1] = make_float4(rw[4], rw[5], rw[6], rw[7]);
                }
                __syncwarp();
                {
                    // lane j: step tw + j of channel c
                    const int t = tw + j;
                    const float dt = sPa[c * kPS + t].x;
                    const float2 pb = sPb[c * kPS + t];   // dy, dout*silu'(z)
                    const float2 uv = sU[c * kPS + t];
                    const float dd = fmaf(uv.x, GB, Q) * uv.y;
                    dbias += dd;
                    dDacc = fmaf(pb.x, uv.x, dDacc);
                    sPa[c * kPS + t] = make_float2(fmaf(dt, GB, pb.x * Dc), dd);
                    sPb[c * kPS + t].x = fmaf(Dc, uv.x, yw) * pb.y;
                }
            }
            // the block's du, ddelta, dz rows of this warp's channels (lane = step)
            __syncwarp();
            if (t0 + lane < L) {
                using R = typename Io<T>::raw;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int cc = warp * 4 + i;
                    const float2 o = sPa[cc * kPS + lane];
                    const int64_t at = (row0 + cc) * L + t0 + lane;
                    static_cast<R*>(p.du)[at] = Io<T>::from(o.x);
                    static_cast<R*>(p.ddelta)[at] = Io<T>::from(o.y);
                    if (zz) static_cast<R*>(p.dz)[at] = Io<T>::from(sPb[cc * kPS + lane].x);
                }
            }
        }

        // the last block's dB, dC terms
        __syncthreads();
        red_add<NW>(sR, dBg, dCg, (int64_t)blk0 * kBT, L, rvec, tid);
        // hand the state gradient to the segment before; this segment's parameter partials
        *reinterpret_cast<float2*>(p.carry2 + (us * kCT + c) * kN + 2 * j) = gs;
        if (seg == 0 && p.dh0) *reinterpret_cast<float2*>(p.dh0 + (row0 + c) * kN + 2 * j) = gs;
        *reinterpret_cast<float2*>(p.dAp + ((int64_t)seg * rows + row0 + c) * kN + 2 * j) = dAacc;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            dbias += __shfl_xor_sync(0xffffffffu, dbias, o);
            dDacc += __shfl_xor_sync(0xffffffffu, dDacc, o);
        }
        if (j == 0) {
            p.dbp[(int64_t)seg * rows + row0 + c] = dbias;
            p.dDp[(int64_t)seg * rows + row0 + c] = dDacc;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            st_release(p.flag2 + us, 1u);
        }
    }
}

// dA, dD, dbias: sums over batch rows and segments of the per-row partials, in a fixed
// order (dB and dC were added by the first kernel).
__global__ void __launch_bounds__(256) scan_bwd_finalize(const BwdParams p, float* dA, float* dD, float* dbias) {
    const int64_t Dm = p.dim;
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = p.batch * Dm;
    if (k < Dm * kN) {
        float s = 0.f;
        for (int64_t b = 0; b < p.batch; ++b)
            for (int sg = 0; sg < p.nseg; ++sg) s += p.dAp[(sg * rows + b * Dm) * kN + k];
        dA[k] = s;
        return;
    }
    const int64_t e = k - Dm * kN;
    if (e < 2 * Dm) {
        const bool isb = e >= Dm;
        const int64_t dd = isb ? e - Dm : e;
        float* dst = isb ? dbias : dD;
        if (!dst) return;
        const float* src = isb ? p.dbp : p.dDp;
        float s = 0.f;
        for (int64_t b = 0; b < p.batch; ++b)
            for (int sg = 0; sg < p.nseg; ++sg) s += src[sg * rows + b * Dm + dd];
        dst[dd] = s;
    }
}

// The schedule: persistent CTAs (as many as fit at once, at most one per forward unit)
// and the cut of each tile's sequence into segments, about 8 units per CTA and pass.
struct Sched {
    int ctas, nseg, seg_blocks;
    int nw, ct;   // warps per CTA and channels per tile
};

Sched make_sched(const ssm_dims_t& d, int sms, int per_sm, int nw) {
    const int ct = 4 * nw;
    const int64_t ntiles = d.batch * d.dim / ct;
    const int64_t nblk = (d.seqlen + kBT - 1) / kBT;
    const int64_t slots = (int64_t)sms * per_sm;
    int64_t want = (8 * slots + ntiles - 1) / ntiles;          // segments per tile
    int64_t sb = (nblk + want - 1) / (want > 0 ? want : 1);
    if (sb < 4) sb = 4;                                          // at least 128 steps per unit
    if (sb > nblk) sb = nblk > 0 ? nblk : 1;
    Sched s;
    s.nw = nw;
    s.ct = ct;
    s.seg_blocks = (int)sb;
    s.nseg = (int)((nblk + sb - 1) / sb);
    const int64_t units = ntiles * s.nseg;
    s.ctas = (int)(units < slots ? units : slots);
    return s;
}

struct WsLayout {
    int64_t ticket, flag1, flag2, zero_end;        // zeroed before every launch
    int64_t carry1, carry2, ckpt, dAp, dDp, dbp, total;   // byte offsets
};

__host__ int64_t align256(int64_t v) { return (v + 255) & ~(int64_t)255; }

WsLayout ws_layout(const ssm_dims_t& d, const Sched& s) {
    const int64_t rows = d.batch * d.dim;
    const int64_t ct = s.ct;
    const int64_t ntiles = rows / ct;
    const int64_t nblk = (d.seqlen + kBT - 1) / kBT;
    const int64_t slots = ntiles * s.nseg;
    WsLayout w;
    w.ticket = 0;                                  // ticket (u32), status (i32)
    w.flag1 = 256;
    w.flag2 = align256(w.flag1 + slots * 4);
    w.zero_end = align256(w.flag2 + slots * 4);
    w.carry1 = w.zero_end;
    w.carry2 = align256(w.carry1 + slots * ct * kN * 4);
    w.ckpt = align256(w.carry2 + slots * ct * kN * 4);
    w.dAp = align256(w.ckpt + ntiles * ct * nblk * kN * 4);
    w.dDp = align256(w.dAp + (int64_t)s.nseg * rows * kN * 4);
    w.dbp = align256(w.dDp + (int64_t)s.nseg * rows * 4);
    w.total = align256(w.dbp + (int64_t)s.nseg * rows * 4);
    return w;
}

// CTAs of the backward kernel that fit on one SM of the current device, and its SM count
// (queried once per device and dtype)
template <typename T, int NW>
bool device_fit(int* sms, int* per_sm) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static int cache[kMaxDev][2];   // {sms, per_sm}; 0 = not queried yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < kMaxDev && cache[dev][0] > 0) {
        *sms = cache[dev][0];
        *per_sm = cache[dev][1];
        return true;
    }
    if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaFuncSetAttribute(scan_bwd_kernel<T, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Smem<T, NW>::TOTAL) != cudaSuccess)
        return false;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, scan_bwd_kernel<T, NW>, Bw<NW>::THREADS,
                                                      Smem<T, NW>::TOTAL) != cudaSuccess)
        return false;
    if (*per_sm < 1) *per_sm = 1;
    if (dev < kMaxDev) {
        cache[dev][0] = *sms;
        cache[dev][1] = *per_sm;
    }
    return true;
}

// The CTA size: 8 warps (32-channel tiles), or 4 warps (16-channel tiles) when the
// 32-channel tiles are fewer than the CTAs that fit at once: each tile's chain of units
// runs in order, so the tiles bound the CTAs at work (one batch row of 5120 channels: 160
// tiles against 296 slots).
bool plan_for(const ssm_dims_t& d, Sched* s, WsLayout* w) {
    const bool bf = d.io_dtype == SSM_BF16;
    int sms = 0, per_sm = 0;
    if (!(bf ? device_fit<__nv_bfloat16, 8>(&sms, &per_sm) : device_fit<float, 8>(&sms, &per_sm))) return false;
    int nw = 8;
    if (d.batch * d.dim / 32 < (int64_t)sms * per_sm) {
        nw = 4;
        if (!(bf ? device_fit<__nv_bfloat16, 4>(&sms, &per_sm) : device_fit<float, 4>(&sms, &per_sm))) return false;
    }
    *s = make_sched(d, sms, per_sm, nw);
    *w = ws_layout(d, *s);
    return true;
}

int check_dims(const ssm_dims_t* d) {
    if (!d || d->batch < 0 || d->dim <= 0 || d->seqlen < 0 || d->dstate <= 0 || d->nheads <= 0 || d->ngroups <= 0)
        return SSM_ERR_INVALID_ARG;
    if (d->dim % d->nheads || d->dim % d->ngroups || d->reserved != 0) return SSM_ERR_INVALID_ARG;
    if (d->io_dtype != SSM_F32 && d->io_dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
    if (d->batch > ((int64_t)1 << 40) / d->dim || (d->seqlen > 0 && d->batch * d->dim > ((int64_t)1 << 40) / d->seqlen))
        return SSM_ERR_INVALID_ARG;
    // what the kernel covers: the S6 layout, dstate 16, whole 32-channel tiles inside a group
    if (d->nheads != d->dim || d->dstate != kN || (d->dim / d->ngroups) % 32 != 0) return SSM_ERR_UNSUPPORTED;
    if (d->batch * d->dim / 16 > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

template <typename T, int NW>
int launch(const BwdParams& prm, float* dA, float* dD, float* dbias, int ctas, cudaStream_t s) {
    constexpr int smem = Smem<T, NW>::TOTAL;
    scan_bwd_kernel<T, NW><<<(unsigned)ctas, Bw<NW>::THREADS, smem, s>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
    const int64_t work = prm.dim * kN + 2 * prm.dim;
    const int64_t blocks = (work + 255) / 256;
    if (blocks > 0x7FFFFFFF) return SSM_ERR_UNSUPPORTED;
    scan_bwd_finalize<<<(unsigned)blocks, 256, 0, s>>>(prm, dA, dD, dbias);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // namespace
}  // namespace ssm

// test hooks (process-wide): a stall makes every wait of a chained unit wait for a flag
// value nobody writes, so it runs out and the call reports SSM_ERR_TIMEOUT
static unsigned g_hook_stall = 0;
static uint64_t g_hook_budget_ns = 0;

extern "C" int ssm_selective_scan_bwd_test_hooks(int stall, int64_t wait_budget_us) {
    if (wait_budget_us < 0 || wait_budget_us > 10000000) return SSM_ERR_INVALID_ARG;
    g_hook_stall = stall ? 1u : 0u;
    g_hook_budget_ns = (uint64_t)wait_budget_us * 1000ull;
    return SSM_OK;
}

extern "C" int ssm_selective_scan_bwd_workspace_size(const ssm_dims_t* dims, size_t* bytes) {
    using namespace ssm;
    if (!bytes) return SSM_ERR_INVALID_ARG;
    const int rc = check_dims(dims);
    if (rc == SSM_ERR_UNSUPPORTED && bwd_generic_supported(*dims) == SSM_OK) {
        *bytes = (size_t)bwd_generic_workspace_bytes(*dims);
        return SSM_OK;
    }
    if (rc != SSM_OK) return rc;
    Sched sc;
    WsLayout w;
    if (!plan_for(*dims, &sc, &w)) return SSM_ERR_CUDA;
    *bytes = (size_t)w.total;
    return SSM_OK;
}

extern "C" int ssm_selective_scan_bwd_device_status(void* workspace, ssm_stream_t stream) {
    if (!workspace) return SSM_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int st = SSM_OK;
    int* status = reinterpret_cast<int*>(static_cast<unsigned char*>(workspace) + 4);
    if (cudaMemcpyAsync(&st, status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (st != SSM_OK && cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return SSM_ERR_CUDA;
    return st;
}

extern "C" int ssm_selective_scan_bwd(const ssm_dims_t* dims, const void* u, const void* delta, const float* A,
                                      const void* B, const void* C, const float* D, const void* z,
                                      const float* delta_bias, int softplus, const float* h0, const void* dout,
                                      const float* dlast, const ssm_grads_t* grads, void* workspace,
                                      size_t workspace_bytes, ssm_stream_t stream) {
    return ssm_selective_scan_bwd_ckpt(dims, u, delta, A, B, C, D, z, delta_bias, softplus, h0, dout, dlast, nullptr,
                                       grads, workspace, workspace_bytes, stream);
}

extern "C" int ssm_selective_scan_bwd_ckpt(const ssm_dims_t* dims, const void* u, const void* delta, const float* A,
                                           const void* B, const void* C, const float* D, const void* z,
                                           const float* delta_bias, int softplus, const float* h0,
                                           const void* dout, const float* dlast, const float* ckpt,
                                           const ssm_grads_t* grads, void* workspace, size_t workspace_bytes,
                                           ssm_stream_t stream) {
    using namespace ssm;
    const int rc = check_dims(dims);
    // the shapes the tiled kernel does not take (per-head layout, dstate other than 16, tiles
    // that do not divide a group) run on the generic backward
    const bool generic = rc == SSM_ERR_UNSUPPORTED && bwd_generic_supported(*dims) == SSM_OK;
    if (rc != SSM_OK && !generic) return rc;
    if (!grads || !grads->dA) return SSM_ERR_INVALID_ARG;
    if (generic && ckpt) return SSM_ERR_INVALID_ARG;   // the forward stores states only for the tiled kernel's shapes
    if (dims->batch == 0 || dims->seqlen == 0) {
        // no steps (the per-step tensors are empty and may be NULL): every gradient is zero, dh0 = dlast
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        const int64_t N = dims->dstate;
        const int64_t rows = dims->batch * dims->dim, esz = dims->io_dtype == SSM_BF16 ? 2 : 4;
        const int64_t nbc = dims->batch * dims->ngroups * N * dims->seqlen * 4;
        const int64_t nA = dims->nheads != dims->dim ? dims->nheads : dims->dim * N;
        bool ok = cudaMemsetAsync(grads->dA, 0, nA * 4, s) == cudaSuccess;
        if (workspace && workspace_bytes >= 8) ok = ok && cudaMemsetAsync(workspace, 0, 8, s) == cudaSuccess;
        if (grads->dD) ok = ok && cudaMemsetAsync(grads->dD, 0, dims->dim * 4, s) == cudaSuccess;
        if (grads->ddelta_bias) ok = ok && cudaMemsetAsync(grads->ddelta_bias, 0, dims->nheads * 4, s) == cudaSuccess;
        if (nbc) ok = ok && cudaMemsetAsync(grads->dB, 0, nbc, s) == cudaSuccess &&
                      cudaMemsetAsync(grads->dC, 0, nbc, s) == cudaSuccess;
        if (rows > 0 && dims->seqlen > 0) {
            ok = ok && cudaMemsetAsync(grads->du, 0, rows * dims->seqlen * esz, s) == cudaSuccess &&
                 cudaMemsetAsync(grads->ddelta, 0, dims->batch * dims->nheads * dims->seqlen * esz, s) == cudaSuccess;
            if (grads->dz) ok = ok && cudaMemsetAsync(grads->dz, 0, rows * dims->seqlen * esz, s) == cudaSuccess;
        }
        if (grads->dh0 && rows) {
            ok = ok && (dlast ? cudaMemcpyAsync(grads->dh0, dlast, rows * N * 4, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(grads->dh0, 0, rows * N * 4, s)) == cudaSuccess;
        }
        return ok ? SSM_OK : SSM_ERR_CUDA;
    }
    if (!u || !delta || !A || !B || !C || !dout) return SSM_ERR_INVALID_ARG;
    if (!grads->du || !grads->ddelta || !grads->dB || !grads->dC) return SSM_ERR_INVALID_ARG;
    if (z && !grads->dz) return SSM_ERR_INVALID_ARG;
    if (generic) {
        if (!workspace || workspace_bytes < (size_t)bwd_generic_workspace_bytes(*dims)) return SSM_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SSM_ERR_UNSUPPORTED;
        return bwd_generic_launch(*dims, u, delta, A, B, C, D, z, delta_bias, softplus, h0, dout, dlast, *grads,
                                  static_cast<unsigned char*>(workspace), reinterpret_cast<cudaStream_t>(stream));
    }
    Sched sc;
    WsLayout w;
    if (!plan_for(*dims, &sc, &w)) return SSM_ERR_CUDA;
    if (!workspace || workspace_bytes < (size_t)w.total) return SSM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(A) & 7u) ||
        (h0 && (reinterpret_cast<uintptr_t>(h0) & 7u)) || (dlast && (reinterpret_cast<uintptr_t>(dlast) & 7u)) ||
        (grads->dh0 && (reinterpret_cast<uintptr_t>(grads->dh0) & 7u)) ||
        (ckpt && (reinterpret_cast<uintptr_t>(ckpt) & 7u)))
        return SSM_ERR_UNSUPPORTED;
    BwdParams prm;
    prm.u = u; prm.delta = delta; prm.z = z; prm.dout = dout; prm.B = B; prm.C = C;
    prm.A = A; prm.D = D; prm.bias = delta_bias; prm.h0 = h0; prm.dlast = dlast;
    prm.du = grads->du; prm.ddelta = grads->ddelta; prm.dz = grads->dz; prm.dh0 = grads->dh0;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    prm.ticket = reinterpret_cast<unsigned*>(ws + w.ticket);
    prm.status = reinterpret_cast<int*>(ws + w.ticket + 4);
    prm.flag1 = reinterpret_cast<unsigned*>(ws + w.flag1);
    prm.flag2 = reinterpret_cast<unsigned*>(ws + w.flag2);
    prm.carry1 = reinterpret_cast<float*>(ws + w.carry1);
    prm.carry2 = reinterpret_cast<float*>(ws + w.carry2);
    // the forward's states when given (read only), else the kernel's own checkpoints in the workspace
    prm.ckpt = ckpt ? const_cast<float*>(ckpt) : reinterpret_cast<float*>(ws + w.ckpt);
    prm.ext_ckpt = ckpt ? 1 : 0;
    prm.dB = static_cast<float*>(grads->dB);
    prm.dC = static_cast<float*>(grads->dC);
    prm.red_vec = dims->seqlen % 4 == 0 &&
                  ((reinterpret_cast<uintptr_t>(grads->dB) | reinterpret_cast<uintptr_t>(grads->dC)) & 15u) == 0;
    prm.dAp = reinterpret_cast<float*>(ws + w.dAp);
    prm.dDp = reinterpret_cast<float*>(ws + w.dDp);
    prm.dbp = reinterpret_cast<float*>(ws + w.dbp);
    prm.batch = dims->batch; prm.dim = dims->dim; prm.seqlen = dims->seqlen; prm.ngroups = dims->ngroups;
    prm.tiles_per_row = (int)(dims->dim / sc.ct);
    prm.ntiles = dims->batch * dims->dim / sc.ct;
    prm.nseg = sc.nseg;
    prm.seg_blocks = sc.seg_blocks;
    prm.softplus = softplus ? 1 : 0;
    prm.budget_ns = g_hook_budget_ns ? g_hook_budget_ns : 1000000000ull;   // 1 s per wait
    prm.need = g_hook_stall ? 2u : 1u;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the ticket, the status word and the segment flags start at zero (the status of this
    // call is read, and cleared, by ssm_selective_scan_bwd_device_status)
    // dB and dC are sums of atomic adds: they start at zero
    const size_t nbc = (size_t)(dims->batch * dims->ngroups * kN * dims->seqlen) * 4;
    if (cudaMemsetAsync(ws + w.ticket, 0, 8, s) != cudaSuccess ||
        cudaMemsetAsync(ws + w.flag1, 0, (size_t)(w.zero_end - w.flag1), s) != cudaSuccess ||
        cudaMemsetAsync(grads->dB, 0, nbc, s) != cudaSuccess || cudaMemsetAsync(grads->dC, 0, nbc, s) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (dims->io_dtype == SSM_BF16)
        return sc.nw == 8 ? launch<__nv_bfloat16, 8>(prm, grads->dA, grads->dD, grads->ddelta_bias, sc.ctas, s)
                          : launch<__nv_bfloat16, 4>(prm, grads->dA, grads->dD, grads->ddelta_bias, sc.ctas, s);
    return sc.nw == 8 ? launch<float, 8>(prm, grads->dA, grads->dD, grads->ddelta_bias, sc.ctas, s)
                      : launch<float, 4>(prm, grads->dA, grads->dD, grads->ddelta_bias, sc.ctas, s);
}
