// ssd_bwd_tc.cu -- the chunk sums and the per-chunk gradients of one scan
// direction on the tensor core (bf16 io, headdim 64, d_state 128, one B/C
// group), in 128-position chunks.
//
// The derivative and its chunked evaluation are those of ssd_bwd.cu (the scan
// is trained inside the DiffuMamba backbone, technical summary section 2):
// with cs the cumulative A dt of a chunk in scan order,
//
//   chunk sums:  sf_c = sum_k exp(cl - cs_k) dt_k x_k (outer) B_k,  sg_c = sum_k exp(cs_k) gy_k (outer) C_k
//   per chunk, with Sin / Gin the state / adjoint entering the chunk (after the passes):
//     g_k   = sum_{s >= k} E[s][k] gy_s + exp(cl - cs_k) Gin B_k,   E[k][s] = (C_k.B_s) exp(cs_k - cs_s), s <= k
//     dx_k  = dt_k g_k + D gy_k,                                    u_k = x_k . g_k
//     dB_k  = dt_k (sum_{s >= k} F[k][s] C_s + exp(cl - cs_k) Gin^T x_k),  F[k][s] = (x_k.gy_s) exp(cs_s - cs_k)
//     dC_k  = sum_{s <= k} F[s][k] dt_s B_s + exp(cs_k) Sin^T gy_k
//     <gy_k, y_k - D x_k> = sum_{s <= k} E[k][s] dt_s (x_s.gy_k) + exp(cs_k) C_k . (Sin^T gy_k)
//
// The pair products C.B^T, B.C^T, x.gy^T and gy.x^T are exact in float32 from
// bf16 inputs and run on the tensor core into TMEM.  The CUDA cores weight
// them with the exact per-element decays and causal masks, in place, and the
// weighted matrices are the A operands (from TMEM) of the output products.
// Every float32 operand that is not an input (the weighted pair matrices, the
// chunk states, the weighted rows of the chunk sums) enters as two bf16 terms,
// hi = bf16(v) and lo = bf16(v - hi), each its own MMA: about 16 significant
// bits, so the gradients keep the float32 path's accuracy.
//
// dB and dC of the one B/C group are the sums over the heads: each CTA adds its head's part
// into the (zeroed) outputs with vector float32 reductions in L2, so no per-head copy reaches
// DRAM; the order of the additions varies, so dB and dC can differ between runs in the last
// bits.
//
// Rows: a chunk is 128 consecutive tokens loaded by TMA in memory order; scan
// position k of memory row r is r forward, 127 - r reverse.  One CTA per
// (chunk, head, batch row); every barrier completes once (parity 0), every
// wait is bounded and records SSD_ERR_TIMEOUT in the status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "ssd_internal.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr uint32_t kTile = kQ * 64 * 2;       // [128 rows][64] bf16, 128-byte swizzled: 16 KB
constexpr uint32_t kHalf = 64 * 64 * 2;       // [64 rows][64] bf16: 8 KB (half of a [p][n] state)
constexpr float kLog2e = 1.4426950408889634f;

struct BwdTcMaps {
    CUtensorMap x, gy, b, c;
};

struct BwdTcParams {
    int batch, L, H, nc, dir;
    const __nv_bfloat16 *dt;
    const float *A, *D;
    float *sf, *sg, *dec;                     // chunk sums in, states after the passes (per chunk)
    float *gx, *gB, *gC, *gcs, *u, *gxd;      // gB, gC: [batch][L][N], zeroed, summed over heads here
    int *status;
    long long wait_cycles;
};

__device__ __forceinline__ size_t slot_of(const BwdTcParams &p, int b, int h, int c) {
    return (((size_t)b * p.nc + c) * p.H + h) * (size_t)(kP * kN);
}

// v -> (hi, lo) bf16 pairs: hi = bf16(v), lo = bf16(v - hi)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(a, b);
    lo = pack_bf16(a - bf16lo(hi), b - bf16hi(hi));
}

// A [64 p][128 n] float32 state, row-major, into hi and lo bf16 tiles: each is two swizzled
// [64][64] halves (n 0-63, n 64-127).  Threads 0 .. NTHR - 1 share the work.
template <int NTHR>
__device__ __forceinline__ void stage_state(const float *src, uint8_t *hi, uint8_t *lo, int tid) {
    constexpr int kIt = kP * kN / 8 / NTHR;
    static_assert(kIt * NTHR * 8 == kP * kN, "state staging");
    float4 v[kIt][2];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {      // every load in flight before the first conversion
        const int i = tid + NTHR * it;
        v[it][0] = *reinterpret_cast<const float4 *>(src + (size_t)i * 8);
        v[it][1] = *reinterpret_cast<const float4 *>(src + (size_t)i * 8 + 4);
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int i = tid + NTHR * it;
        const int p = i / (kN / 8), n8 = (i % (kN / 8)) * 8;
        const float4 v0 = v[it][0], v1 = v[it][1];
        uint4 h, l;
        split2(v0.x, v0.y, h.x, l.x);
        split2(v0.z, v0.w, h.y, l.y);
        split2(v1.x, v1.y, h.z, l.z);
        split2(v1.z, v1.w, h.w, l.w);
        const uint32_t off = (n8 >> 6) * kHalf + swz(p, (n8 & 63) >> 3);
        *reinterpret_cast<uint4 *>(hi + off) = h;
        *reinterpret_cast<uint4 *>(lo + off) = l;
    }
}

// ------------------------------------------------------------------ chunk sums

// smem: x (16 KB) | gy | B (2 halves) | C (2 halves) | w x hi | w x lo | e gy hi | e gy lo | tables
constexpr uint32_t kSX = 0, kSG = kTile, kSB = 2 * kTile, kSC = 4 * kTile, kSWXH = 6 * kTile, kSWXL = 7 * kTile,
                   kSEGH = 8 * kTile, kSEGL = 9 * kTile, kSTab = 10 * kTile;
constexpr uint32_t kSBar = kSTab + 4 * kQ * 4;
enum SumsBar { SB_FULL = 0, SB_READY, SB_DONE, SB_TAB, kSumsBars };
constexpr uint32_t kSMisc = kSBar + kSumsBars * 8;
constexpr uint32_t kSumsSmem = kSMisc + 32 + 1024;
constexpr int kSumsThreads = 192;              // warps 0-3 rows, warp 4 loads, warp 5 MMA

__global__ void __launch_bounds__(kSumsThreads, 1) k_bwd_tc_sums(const __grid_constant__ BwdTcMaps maps,
                                                                 const __grid_constant__ BwdTcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kSBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kSMisc + 4);
    float *tab = reinterpret_cast<float *>(sm + kSTab);   // [0,128) w by memory row, [128,256) e, [256] cl
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int L = prm.L, dir = prm.dir;
    const int row0 = b * L + (dir > 0 ? c * kQ : L - (c + 1) * kQ);   // first token row of the chunk
    const uint32_t MASK = 0xffffffffu;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kSumsBars; ++i) mbar_init(bar(i), i == SB_READY ? 4 : 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            mbar_expect_tx(bar(SB_FULL), 6 * kTile);
            tma_load_2d(sbase + kSX, &maps.x, h * kP, row0, bar(SB_FULL));
            tma_load_2d(sbase + kSG, &maps.gy, h * kP, row0, bar(SB_FULL));
            for (int q = 0; q < 2; ++q) {
                tma_load_2d(sbase + kSB + q * kTile, &maps.b, q * 64, row0, bar(SB_FULL));
                tma_load_2d(sbase + kSC + q * kTile, &maps.c, q * 64, row0, bar(SB_FULL));
            }
            if (!mbar_wait(bar(SB_FULL), 0, 1u, abort_flag, prm.status, 91)) mbar_drain(bar(SB_FULL), 0, prm.wait_cycles);
        }
        __syncwarp();
    } else if (warp == 5) {
        // acc_f [n][p] = sum_r B[r][n] (w x)[r][p]  (A = B^T, M = n; both operands MN-major),
        // acc_g [n][p] = sum_r C[r][n] (e gy)[r][p]; hi then lo
        bool ok = mbar_wait(bar(SB_FULL), 0, MASK, abort_flag, prm.status, 92) &&
                  mbar_wait(bar(SB_READY), 0, MASK, abort_flag, prm.status, 93);
        if (ok) {
            tc_fence_after();
            const uint32_t id = idesc(64, 1, 1);
            const SDesc dB = make_sdesc(sbase + kSB, kTile, 1024), dC = make_sdesc(sbase + kSC, kTile, 1024);
            const SDesc w[4] = {make_sdesc(sbase + kSWXH, kTile, 1024), make_sdesc(sbase + kSWXL, kTile, 1024),
                                make_sdesc(sbase + kSEGH, kTile, 1024), make_sdesc(sbase + kSEGL, kTile, 1024)};
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem, dB.at(ks * 2048), w[t].at(ks * 2048), id, t | ks);
#pragma unroll
            for (int t = 2; t < 4; ++t)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss_w(tmem + 64, dC.at(ks * 2048), w[t].at(ks * 2048), id, (t - 2) | ks);
        }
        mma_commit_w(bar(SB_DONE));
        if (lane == 0 && !ok) mbar_drain(bar(SB_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // warps 0-3: thread r = memory row r of the chunk.  Warp 0 forms the weights first.
        const int r = threadIdx.x;
        const float A2 = prm.A[h] * kLog2e;
        if (warp == 0) {
            // scan positions lane + 32 t; inclusive prefix sums of dt in scan order
            float d[4], incl[4], col[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int k = lane + 32 * t;
                const int tr = row0 + (dir > 0 ? k : kQ - 1 - k);
                d[t] = __bfloat162float(prm.dt[(size_t)tr * prm.H + h]);
                incl[t] = d[t];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(MASK, incl[t], o);
                    if (lane >= o) incl[t] += v;
                }
                col[t] = __shfl_sync(MASK, incl[t], 31);
            }
            const float total = col[0] + col[1] + col[2] + col[3];
            float before = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int k = lane + 32 * t;
                const int mr = dir > 0 ? k : kQ - 1 - k;
                const float cs2 = A2 * (before + incl[t]);
                tab[mr] = ex2_ftz(A2 * total - cs2) * d[t];       // exp(cl - cs_k) dt_k
                tab[kQ + mr] = ex2_ftz(cs2);                       // exp(cs_k)
                before += col[t];
            }
            if (lane == 0) tab[2 * kQ] = ex2_ftz(A2 * total);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(SB_TAB));
        }
        bool ok = mbar_wait(bar(SB_TAB), 0, MASK, abort_flag, prm.status, 94) &&
                  mbar_wait(bar(SB_FULL), 0, MASK, abort_flag, prm.status, 95);
        if (ok) {
            const float w = tab[r], e = tab[kQ + r];
            const uint8_t *xs = sm + kSX, *gs = sm + kSG;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + swz(r, q));
                const uint4 gv = *reinterpret_cast<const uint4 *>(gs + swz(r, q));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
                uint32_t hx[4], lx[4], hg[4], lg[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    split2(bf16lo(xw[i]) * w, bf16hi(xw[i]) * w, hx[i], lx[i]);
                    split2(bf16lo(gw[i]) * e, bf16hi(gw[i]) * e, hg[i], lg[i]);
                }
                *reinterpret_cast<uint4 *>(sm + kSWXH + swz(r, q)) = make_uint4(hx[0], hx[1], hx[2], hx[3]);
                *reinterpret_cast<uint4 *>(sm + kSWXL + swz(r, q)) = make_uint4(lx[0], lx[1], lx[2], lx[3]);
                *reinterpret_cast<uint4 *>(sm + kSEGH + swz(r, q)) = make_uint4(hg[0], hg[1], hg[2], hg[3]);
                *reinterpret_cast<uint4 *>(sm + kSEGL + swz(r, q)) = make_uint4(lg[0], lg[1], lg[2], lg[3]);
            }
            fence_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(SB_READY));
        if (ok && mbar_wait(bar(SB_DONE), 0, MASK, abort_flag, prm.status, 96)) {
            tc_fence_after();
            // TMEM lane quarter = warp: rows n = 32 warp + lane; columns p of acc_f, then acc_g
            const int n = 32 * warp + lane;
            const size_t slot = slot_of(prm, b, h, c);
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
            float v[32];
            for (int half = 0; half < 4; ++half) {
                tmem_ld32(ta + 32 * half, v);
                float *dst = (half < 2 ? prm.sf : prm.sg) + slot;
                const int p0 = 32 * (half & 1);
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[(size_t)(p0 + i) * kN + n] = v[i];
            }
            if (r == 0) prm.dec[((size_t)b * prm.H + h) * prm.nc + c] = tab[2 * kQ];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
    }
}

// ------------------------------------------------------------------ per-chunk gradients

// smem: x | gy | B (2 halves) | C (2 halves) | Gin hi | Gin lo | Sin hi | Sin lo (each [64][128] as two
// 8 KB halves) | tables | partial sums
constexpr uint32_t kCX = 0, kCG = kTile, kCB = 2 * kTile, kCC = 4 * kTile, kCGH = 6 * kTile,
                   kCGL = kCGH + 2 * kHalf, kCSH = kCGL + 2 * kHalf, kCSL = kCSH + 2 * kHalf,
                   kCTab = kCSL + 2 * kHalf;
// tables (floats, by memory row): c2 (log2 cs), dt, exp(cl - cs), exp(cs)
// partials [4 column groups][128]: u, red2, red2b; the diagonal <gy_k, x_k> [128]; its 4 warp sums
constexpr uint32_t kCPart = kCTab + 4 * kQ * 4;
// dx of the chunk, [128 rows][64 p] float32 with rows kDxS floats apart, for coalesced stores
constexpr int kDxS = kP + 4;
constexpr uint32_t kCDx = kCPart + (3 * 4 * kQ + kQ + 4) * 4;
constexpr uint32_t kCBar = (kCDx + kQ * kDxS * 4 + 7) / 8 * 8;
enum ChunkBar { CB_FULL = 0, CB_TAB, CB_SREADY, CB_PA, CB_PB, CB_C1, CB_GREAD, CB_C2, CB_DBREAD, CB_C3, CB_FIN,
                CB_DX, kChunkBars };
constexpr uint32_t kCMisc = kCBar + kChunkBars * 8;
constexpr uint32_t kChunkSmem = kCMisc + 32 + 1024;
constexpr int kChunkThreads = 576;             // warps 0-15 CUDA cores, 16 loads, 17 MMA
static_assert(kChunkSmem <= 232448 && kSumsSmem <= 232448, "shared memory");

// TMEM regions (columns): the four pair products, then the output accumulators in their place
constexpr uint32_t kR0 = 0, kR1 = 128, kR2 = 256, kR3 = 384;

__global__ void __launch_bounds__(kChunkThreads, 1) k_bwd_tc_chunk(const __grid_constant__ BwdTcMaps maps,
                                                                   const __grid_constant__ BwdTcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kCBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kCMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kCMisc + 4);
    float *c2t = reinterpret_cast<float *>(sm + kCTab), *dtt = c2t + kQ, *elt = dtt + kQ, *ekt = elt + kQ;
    float *pu = reinterpret_cast<float *>(sm + kCPart), *pr2 = pu + 4 * kQ, *pr2b = pr2 + 4 * kQ, *pdg = pr2b + 4 * kQ,
          *pdw = pdg + kQ;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int L = prm.L, dir = prm.dir;
    const int row0 = b * L + (dir > 0 ? c * kQ : L - (c + 1) * kQ);
    const uint32_t MASK = 0xffffffffu;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kChunkBars; ++i) {
            uint32_t cnt = 1;
            if (i == CB_SREADY || i == CB_PB || i == CB_GREAD || i == CB_DBREAD || i == CB_FIN || i == CB_DX) cnt = 16;
            mbar_init(bar(i), cnt);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 17) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 16) {
        if (lane == 0) {
            mbar_expect_tx(bar(CB_FULL), 6 * kTile);
            tma_load_2d(sbase + kCX, &maps.x, h * kP, row0, bar(CB_FULL));
            tma_load_2d(sbase + kCG, &maps.gy, h * kP, row0, bar(CB_FULL));
            for (int q = 0; q < 2; ++q) {
                tma_load_2d(sbase + kCB + q * kTile, &maps.b, q * 64, row0, bar(CB_FULL));
                tma_load_2d(sbase + kCC + q * kTile, &maps.c, q * 64, row0, bar(CB_FULL));
            }
            if (!mbar_wait(bar(CB_FULL), 0, 1u, abort_flag, prm.status, 101)) mbar_drain(bar(CB_FULL), 0, prm.wait_cycles);
        }
        __syncwarp();
    } else if (warp == 17) {
        // ---------------------------------------------------------- MMA issue
        const SDesc dXk = make_sdesc(sbase + kCX, kTile, 1024), dGk = make_sdesc(sbase + kCG, kTile, 1024);
        const SDesc dBk = make_sdesc(sbase + kCB, kTile, 1024), dCk = make_sdesc(sbase + kCC, kTile, 1024);
        // K-major (K = n) views of the [p][n] states: rows p, two 8 KB halves along n
        const SDesc dGinH = make_sdesc(sbase + kCGH, kHalf, 1024), dGinL = make_sdesc(sbase + kCGL, kHalf, 1024);
        const SDesc dSinH = make_sdesc(sbase + kCSH, kHalf, 1024), dSinL = make_sdesc(sbase + kCSL, kHalf, 1024);
        const uint32_t id_pair = idesc(128, 0, 0), id_n64_mn = idesc(64, 0, 1), id_n64_k = idesc(64, 0, 0),
                       id_n128_mn = idesc(128, 0, 1);
        bool ok = mbar_wait(bar(CB_FULL), 0, MASK, abort_flag, prm.status, 102);
        if (ok) {
            tc_fence_after();
            // phase A: G = C B^T, Gt = B C^T (K = n, 8 steps); H = x gy^T, Ht = gy x^T (K = p, 4 steps)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * kTile + (ks & 3) * 32;
                mma_ss_w(tmem + kR0, dCk.at(off), dBk.at(off), id_pair, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * kTile + (ks & 3) * 32;
                mma_ss_w(tmem + kR1, dBk.at(off), dCk.at(off), id_pair, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_ss_w(tmem + kR2, dXk.at(ks * 32), dGk.at(ks * 32), id_pair, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_ss_w(tmem + kR3, dGk.at(ks * 32), dXk.at(ks * 32), id_pair, ks > 0);
            mma_commit_w(bar(CB_PA));
        }
        ok = ok && mbar_wait(bar(CB_PB), 0, MASK, abort_flag, prm.status, 103) &&
             mbar_wait(bar(CB_SREADY), 0, MASK, abort_flag, prm.status, 104);
        if (ok) {
            tc_fence_after();
            // C1: g1 = Et gy (A = Et hi/lo in R1, B = gy as N = p, K = s: MN-major) -> R0 [0, 64);
            //     g2 = B Gin^T (A = B rows, K = n; B = Gin as N = p, K = n) -> R0 [64, 128)
            const SDesc dGm = make_sdesc(sbase + kCG, kTile, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_ts_w(tmem + kR0, tmem + kR1 + 16 * ks, dGm.at(ks * 2048), id_n64_mn, ks > 0);
                mma_ts_w(tmem + kR0, tmem + kR1 + 16 * ks + 8, dGm.at(ks * 2048), id_n64_mn, 1);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t oa = (ks >> 2) * kTile + (ks & 3) * 32, ob = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_ss_w(tmem + kR0 + 64, dBk.at(oa), dGinH.at(ob), id_n64_k, ks > 0);
                mma_ss_w(tmem + kR0 + 64, dBk.at(oa), dGinL.at(ob), id_n64_k, 1);
            }
            mma_commit_w(bar(CB_C1));
        }
        // C2: dBa = F C (A = F in R2; B = C as N = n, K = s) -> R1, once C1 has read Et there;
        //     dBb = x Gin (A = x rows, K = p; B = Gin as N = n, K = p) -> R0, once g has been read
        ok = ok && mbar_wait(bar(CB_C1), 0, MASK, abort_flag, prm.status, 105);
        if (ok) {
            tc_fence_after();
            const SDesc dCm = make_sdesc(sbase + kCC, kTile, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_ts_w(tmem + kR1, tmem + kR2 + 16 * ks, dCm.at(ks * 2048), id_n128_mn, ks > 0);
                mma_ts_w(tmem + kR1, tmem + kR2 + 16 * ks + 8, dCm.at(ks * 2048), id_n128_mn, 1);
            }
        }
        ok = ok && mbar_wait(bar(CB_GREAD), 0, MASK, abort_flag, prm.status, 106);
        if (ok) {
            tc_fence_after();
            const SDesc dGinHm = make_sdesc(sbase + kCGH, kHalf, 1024), dGinLm = make_sdesc(sbase + kCGL, kHalf, 1024);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_ss_w(tmem + kR0, dXk.at(ks * 32), dGinHm.at(ks * 2048), id_n128_mn, ks > 0);
                mma_ss_w(tmem + kR0, dXk.at(ks * 32), dGinLm.at(ks * 2048), id_n128_mn, 1);
            }
            mma_commit_w(bar(CB_C2));
        }
        // C3: dCa = Ftd B (A = Ftd in R3; B = B as N = n, K = s) -> R2, once C2 has read F there;
        //     dCb = gy Sin (A = gy rows, K = p; B = Sin as N = n, K = p) -> R0, once dB has been read
        ok = ok && mbar_wait(bar(CB_C2), 0, MASK, abort_flag, prm.status, 107);
        if (ok) {
            tc_fence_after();
            const SDesc dBm = make_sdesc(sbase + kCB, kTile, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_ts_w(tmem + kR2, tmem + kR3 + 16 * ks, dBm.at(ks * 2048), id_n128_mn, ks > 0);
                mma_ts_w(tmem + kR2, tmem + kR3 + 16 * ks + 8, dBm.at(ks * 2048), id_n128_mn, 1);
            }
        }
        ok = ok && mbar_wait(bar(CB_DBREAD), 0, MASK, abort_flag, prm.status, 108);
        if (ok) {
            tc_fence_after();
            const SDesc dSinHm = make_sdesc(sbase + kCSH, kHalf, 1024), dSinLm = make_sdesc(sbase + kCSL, kHalf, 1024);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_ss_w(tmem + kR0, dGk.at(ks * 32), dSinHm.at(ks * 2048), id_n128_mn, ks > 0);
                mma_ss_w(tmem + kR0, dGk.at(ks * 32), dSinLm.at(ks * 2048), id_n128_mn, 1);
            }
        }
        mma_commit_w(bar(CB_C3));               // also when aborting: every issued MMA has completed
        if (lane == 0 && !ok) mbar_drain(bar(CB_C3), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // ---------------------------------------------------------- CUDA cores (warps 0-15)
        const int q = warp & 3, cg = warp >> 2;   // TMEM lane quarter (rows), column group
        const int r = 32 * q + lane;              // memory row of the chunk = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const float A2 = prm.A[h] * kLog2e;
        const float Dh = prm.D ? prm.D[h] : 0.f;
        const size_t slot = slot_of(prm, b, h, c);
        if (warp == 0) {
            // tables by memory row: c2 = cs log2(e), dt, exp(cl - cs), exp(cs)
            float d[4], incl[4], col[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int k = lane + 32 * t;
                const int tr = row0 + (dir > 0 ? k : kQ - 1 - k);
                d[t] = __bfloat162float(prm.dt[(size_t)tr * prm.H + h]);
                incl[t] = d[t];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(MASK, incl[t], o);
                    if (lane >= o) incl[t] += v;
                }
                col[t] = __shfl_sync(MASK, incl[t], 31);
            }
            const float cl2 = A2 * (col[0] + col[1] + col[2] + col[3]);
            float before = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int k = lane + 32 * t;
                const int mr = dir > 0 ? k : kQ - 1 - k;
                const float cs2 = A2 * (before + incl[t]);
                c2t[mr] = cs2;
                dtt[mr] = d[t];
                elt[mr] = ex2_ftz(cl2 - cs2);
                ekt[mr] = ex2_ftz(cs2);
                before += col[t];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(CB_TAB));
        }
        // the entering adjoint and state, split into bf16 hi and lo tiles
        stage_state<512>(prm.sg + slot, sm + kCGH, sm + kCGL, threadIdx.x);
        stage_state<512>(prm.sf + slot, sm + kCSH, sm + kCSL, threadIdx.x);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(CB_SREADY));

        bool ok = mbar_wait(bar(CB_TAB), 0, MASK, abort_flag, prm.status, 111) &&
                  mbar_wait(bar(CB_PA), 0, MASK, abort_flag, prm.status, 112);
        // phase B: columns s = memory rows 32 cg .. 32 cg + 31, in two K-steps of 16
        // lower: s at or before r in scan order (E, Ftd); upper: s at or after (Et, F)
        float red2 = 0.f, diag = 0.f;
        if (ok) {
            tc_fence_after();
            const float c2r = c2t[r];
#pragma unroll 1
            for (int hk = 0; hk < 2; ++hk) {
                const int s0 = 32 * cg + 16 * hk;
                // decay factors of this K-step's 16 columns, first exp(cs_k - cs_s) for s at or before
                // the row in scan order (else 0), later exp(cs_s - cs_k) for s at or after it
                float e16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int s = s0 + i;
                    const bool lower = dir > 0 ? s <= r : s >= r;
                    e16[i] = lower ? ex2_ftz(c2r - c2t[s]) : 0.f;
                }
                float v[16], w[16];
                uint32_t hi[8], lo[8];
                // E (from G, for <gy, y - D x> only) and Ftd = Ht exp(cs_k - cs_s) dt_s, in place of Ht
                tmem_ld16(tl + kR0 + s0, v);
                tmem_ld16(tl + kR3 + s0, w);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const float d0 = dtt[s0 + i], d1 = dtt[s0 + i + 1];
                    red2 = fmaf(v[i] * e16[i], d0 * w[i], red2);
                    red2 = fmaf(v[i + 1] * e16[i + 1], d1 * w[i + 1], red2);
                    split2(w[i] * e16[i] * d0, w[i + 1] * e16[i + 1] * d1, hi[i >> 1], lo[i >> 1]);
                }
                tmem_st8_nw(tl + kR3 + s0, hi);
                tmem_st8_nw(tl + kR3 + s0 + 8, lo);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int s = s0 + i;
                    const bool upper = dir > 0 ? s >= r : s <= r;
                    e16[i] = upper ? ex2_ftz(c2t[s] - c2r) : 0.f;
                }
                // Et = Gt exp(cs_s - cs_k), in place of Gt
                tmem_ld16(tl + kR1 + s0, v);
#pragma unroll
                for (int i = 0; i < 16; i += 2) split2(v[i] * e16[i], v[i + 1] * e16[i + 1], hi[i >> 1], lo[i >> 1]);
                tmem_st8_nw(tl + kR1 + s0, hi);
                tmem_st8_nw(tl + kR1 + s0 + 8, lo);
                // F = H exp(cs_s - cs_k), in place of H; the diagonal H[k][k] = <x_k, gy_k>
                tmem_ld16(tl + kR2 + s0, v);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    if (s0 + i == r) diag = v[i];
                    if (s0 + i + 1 == r) diag = v[i + 1];
                    split2(v[i] * e16[i], v[i + 1] * e16[i + 1], hi[i >> 1], lo[i >> 1]);
                }
                tmem_st8_nw(tl + kR2 + s0, hi);
                tmem_st8_nw(tl + kR2 + s0 + 8, lo);
            }
            tmem_wait_st();
            tc_fence_before();
            pr2[cg * kQ + r] = red2;
            if (r >= 32 * cg && r < 32 * cg + 32) pdg[r] = diag;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(CB_PB));

        // token row of memory row r, and the position's scan index
        const size_t trow = (size_t)row0 + r;
        const float dtr = ok ? dtt[r] : 0.f, el = ok ? elt[r] : 0.f, ek = ok ? ekt[r] : 0.f;
        // C1 read-out: g = g1 + exp(cl - cs_k) g2 over p = 16 cg .. 16 cg + 15; dx, u
        ok = ok && mbar_wait(bar(CB_C1), 0, MASK, abort_flag, prm.status, 113);
        if (ok) {
            tc_fence_after();
            const int p0 = 16 * cg;
            float g1[16], g2[16];
            tmem_ld16(tl + kR0 + p0, g1);
            tmem_ld16(tl + kR0 + 64 + p0, g2);
            tc_fence_before();
            const uint8_t *xs = sm + kCX, *gs = sm + kCG;
            float uacc = 0.f, dx[16];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const int ch = (p0 >> 3) + qq;
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + swz(r, ch));
                const uint4 gv = *reinterpret_cast<const uint4 *>(gs + swz(r, ch));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = 8 * qq + 2 * i + e;
                        const float gg = fmaf(el, g2[j], g1[j]);
                        const float xv_ = e ? bf16hi(xw[i]) : bf16lo(xw[i]);
                        const float gy_ = e ? bf16hi(gw[i]) : bf16lo(gw[i]);
                        dx[j] = fmaf(dtr, gg, Dh * gy_);
                        uacc = fmaf(xv_, gg, uacc);
                    }
                }
            }
            float *dxs = reinterpret_cast<float *>(sm + kCDx) + r * kDxS + p0;
#pragma unroll
            for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4 *>(dxs + j) = make_float4(dx[j], dx[j + 1], dx[j + 2], dx[j + 3]);
            pu[cg * kQ + r] = uacc;
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(bar(CB_GREAD));
            mbar_arrive(bar(CB_DX));
        }
        // dx out: half a warp per row, 256 contiguous bytes (16 lanes x 16 bytes) per row
        if (ok && mbar_wait(bar(CB_DX), 0, MASK, abort_flag, prm.status, 117)) {
            const int t = threadIdx.x, c4 = 4 * (t & 15);
            const float *dxs = reinterpret_cast<const float *>(sm + kCDx);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int rr = (t >> 4) + 32 * i;
                const float4 v = *reinterpret_cast<const float4 *>(dxs + rr * kDxS + c4);
                *reinterpret_cast<float4 *>(prm.gx + (((size_t)row0 + rr) * prm.H + h) * kP + c4) = v;
            }
        }
        // C2 read-out: dB = dt (dBa + exp(cl - cs_k) dBb) over n = 32 cg .. 32 cg + 31
        ok = ok && mbar_wait(bar(CB_C2), 0, MASK, abort_flag, prm.status, 114);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int hk = 0; hk < 2; ++hk) {
                const int n0 = 32 * cg + 16 * hk;
                float va[16], vb[16];
                tmem_ld16(tl + kR1 + n0, va);
                tmem_ld16(tl + kR0 + n0, vb);
                float *dst = prm.gB + trow * kN + n0;    // one group: summed over the heads here
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    red_add_f32x4(dst + j, dtr * fmaf(el, vb[j], va[j]), dtr * fmaf(el, vb[j + 1], va[j + 1]),
                                  dtr * fmaf(el, vb[j + 2], va[j + 2]), dtr * fmaf(el, vb[j + 3], va[j + 3]));
            }
            tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(CB_DBREAD));
        // C3 read-out: dC = dCa + exp(cs_k) dCb; the state part of <gy, y - D x>: exp(cs_k) C_k . dCb
        ok = ok && mbar_wait(bar(CB_C3), 0, MASK, abort_flag, prm.status, 115);
        if (ok) {
            tc_fence_after();
            float rb = 0.f;
#pragma unroll 1
            for (int hk = 0; hk < 2; ++hk) {
                const int n0 = 32 * cg + 16 * hk;
                float va[16], vb[16];
                tmem_ld16(tl + kR2 + n0, va);
                tmem_ld16(tl + kR0 + n0, vb);
                float *dst = prm.gC + trow * kN + n0;
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    red_add_f32x4(dst + j, fmaf(ek, vb[j], va[j]), fmaf(ek, vb[j + 1], va[j + 1]),
                                  fmaf(ek, vb[j + 2], va[j + 2]), fmaf(ek, vb[j + 3], va[j + 3]));
                // C_k . dCb over these 16 n (C row r, 16-byte chunks of its n half)
                const uint8_t *cs_ = sm + kCC + (n0 >> 6) * kTile;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const uint4 cv = *reinterpret_cast<const uint4 *>(cs_ + swz(r, ((n0 & 63) >> 3) + qq));
                    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        rb = fmaf(bf16lo(cw[i]), vb[8 * qq + 2 * i], rb);
                        rb = fmaf(bf16hi(cw[i]), vb[8 * qq + 2 * i + 1], rb);
                    }
                }
            }
            tc_fence_before();
            pr2b[cg * kQ + r] = ek * rb;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(CB_FIN));
        // per position: u, gcs; per chunk: sum of <gy, x>
        if (warp < 4 && ok && mbar_wait(bar(CB_FIN), 0, MASK, abort_flag, prm.status, 116)) {
            float uu = 0.f, rr = 0.f;
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
                uu += pu[g4 * kQ + r];
                rr += pr2[g4 * kQ + r] + pr2b[g4 * kQ + r];
            }
            const size_t ti = trow * prm.H + h;
            prm.u[ti] = uu;
            prm.gcs[ti] = rr - dtr * uu;
            float dsum = pdg[r];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(MASK, dsum, o);
            if (lane == 0) pdw[warp] = dsum;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && !*abort_flag)
        prm.gxd[((size_t)b * prm.H + h) * prm.nc + c] = pdw[0] + pdw[1] + pdw[2] + pdw[3];
    if (warp == 17) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

}  // namespace

bool bwd_tc_supported(const BwdArgs &a, bool bf16) {
    return bf16 && a.P == kP && a.N == kN && a.G == 1 && a.Q == kQ && a.L % kQ == 0 && a.H % 8 == 0 &&
           get_encode() != nullptr;
}

namespace {
bool bwd_maps(const BwdArgs &a, BwdTcMaps &m) {
    memset(&m, 0, sizeof m);
    const uint64_t rows = (uint64_t)a.batch * a.L;
    return make_map(&m.x, a.x, rows, (uint64_t)a.H * kP, 64, true) &&
           make_map(&m.gy, a.gy, rows, (uint64_t)a.H * kP, 64, true) && make_map(&m.b, a.B, rows, kN, 64, true) &&
           make_map(&m.c, a.C, rows, kN, 64, true);
}
BwdTcParams bwd_params(const BwdArgs &a) {
    BwdTcParams p{};
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.nc = a.nc; p.dir = a.dir;
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A; p.D = a.D;
    p.sf = a.sf; p.sg = a.sg; p.dec = a.dec;
    p.gx = a.gx; p.gB = a.gB; p.gC = a.gC; p.gcs = a.gcs; p.u = a.u; p.gxd = a.gxd;
    p.status = a.status; p.wait_cycles = a.wait_cycles;
    return p;
}
}  // namespace

cudaError_t launch_bwd_tc_sums(const BwdArgs &a, cudaStream_t st) {
    BwdTcMaps m;
    if (!bwd_maps(a, m)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_tc_sums, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSumsSmem);
    if (e != cudaSuccess) return e;
    k_bwd_tc_sums<<<dim3(a.nc, a.H, a.batch), kSumsThreads, kSumsSmem, st>>>(m, bwd_params(a));
    return cudaGetLastError();
}

cudaError_t launch_bwd_tc_chunk(const BwdArgs &a, cudaStream_t st) {
    BwdTcMaps m;
    if (!bwd_maps(a, m)) return cudaErrorInvalidValue;
    const size_t bytes = sizeof(float) * (size_t)a.batch * a.L * kN;   // one group
    cudaError_t z = cudaMemsetAsync(a.gB, 0, bytes, st);
    if (z == cudaSuccess) z = cudaMemsetAsync(a.gC, 0, bytes, st);
    if (z != cudaSuccess) return z;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_tc_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kChunkSmem);
    if (e != cudaSuccess) return e;
    k_bwd_tc_chunk<<<dim3(a.nc, a.H, a.batch), kChunkThreads, kChunkSmem, st>>>(m, bwd_params(a));
    return cudaGetLastError();
}

}  // namespace ssd
