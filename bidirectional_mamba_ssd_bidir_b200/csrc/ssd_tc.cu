// ssd_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) path of the SSD scan for
// bf16 io, headdim 64, d_state 128, one B/C group shared by a head pair.
//
// One CTA owns (batch b, head pair {h0, h0+1}, direction) and walks the
// sequence in scan order in blocks of 128 tokens, carrying the float32 state
// of both heads in registers.  Per block (rows r = 0..127 in memory order,
// TMEM lane r = token t0 + r), with cs the cumulative A*dt in scan order:
//
//   G    = C B^T                      tcgen05, shared by both heads   TMEM [0,128)
//   M_h  = G (.) decay_h (.) dt        CUDA cores -> bf16 A operand    TMEM [128,256)
//   S^T  = B^T (w (.) X)               tcgen05, N = 2 heads x 64       TMEM [256,384)
//   Y    = C S'^T_prev                 tcgen05, N = 2 heads x 64       TMEM [384,512)
//   Y   *= exp(cs_r) per row           CUDA cores (TMEM ld/st)
//   Y   += M_h X_h                     tcgen05, A from TMEM, N = 64
//   y    = Y + D x                     CUDA cores -> bf16 global stores
//   S'   = exp(cs_last) S' + S         CUDA cores, float32 registers -> bf16 smem
//
// This is the chunked evaluation of the recurrence S <- exp(dt A) S +
// dt x (outer) B, y = C.S + D x that the Mamba-2 layers of the DiffuMamba mixer
// ("DiffuMamba", technical summary, section 2) and the R2LM right-to-left
// stream ("Bifocal Diffusion Language Models", section 2, mechanism) run.
// The reverse direction walks the blocks from the end and uses suffix sums
// and the upper triangle: the flip lives in the address arithmetic only.
//
// Warp roles (384 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs (one thread), warps 4-7 do the CUDA-core work of head h0
// and warps 8-11 that of head h0+1 (thread r <-> TMEM lane r).  Every
// mbarrier wait is bounded; a wait that runs out records SSD_ERR_TIMEOUT in
// the status word and the CTA winds down without touching more data.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ssd_tc.cuh"

namespace ssd {
namespace {

constexpr int kBlk = 128;            // tokens per block (MMA M)
constexpr int kP = 64, kN = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTileBytes = kBlk * 64 * 2;        // one [128][64] bf16 swizzled tile = 16 KB

// TMEM column map
constexpr uint32_t kColG = 0, kColM = 128, kColS = 256, kColY = 384;

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffX = 0;                          // 2 stages x 2 heads x 16 KB
constexpr uint32_t kOffB = kOffX + 2 * 2 * kTileBytes; // 2 sub-tiles (n 0..63, 64..127)
constexpr uint32_t kOffC = kOffB + 2 * kTileBytes;
constexpr uint32_t kOffWX = kOffC + 2 * kTileBytes;    // 2 heads
constexpr uint32_t kOffSP = kOffWX + 2 * kTileBytes;   // 2 heads, rows = state index n
constexpr uint32_t kOffCS = kOffSP + 2 * kTileBytes;   // float cs2[2][128], dt[2][128]
constexpr uint32_t kOffRed = kOffCS + 4 * kBlk * 4;    // per-WG cross-warp scan scratch
constexpr uint32_t kOffBar = kOffRed + 2 * 8 * 4;
constexpr uint32_t kNumBars = 20;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

enum Bar {
    B_XFULL0 = 0, B_XFULL1, B_XEMPTY0, B_XEMPTY1, B_BCFULL, B_BCEMPTY, B_GFULL, B_GEMPTY,
    B_WXREADY, B_SFULL, B_SEMPTY, B_SPREADY, B_YOFFFULL, B_MREADY, B_RSREADY, B_YFULL, B_YEMPTY, B_DONE, B_WG0, B_WG1
};

constexpr long long kWaitCycles = 4000000000LL;        // ~2 s at B200 clocks
constexpr float kLog2e = 1.4426950408889634f;

// Optional phase timeline for profiling builds (-DSSD_TRACE): %globaltimer
// stamps of CTA 0, first kTraceBlocks blocks, per role and phase.
#ifdef SSD_TRACE
constexpr int kTraceBlocks = 8, kTracePts = 16;
__device__ unsigned long long g_trace[3][kTraceBlocks][kTracePts];
__device__ __forceinline__ void trace_pt(int role, int j, int k) {
    if (blockIdx.x == 0 && j < kTraceBlocks) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_trace[role][j][k] = t;
    }
}
#define SSD_TRACE_PT(role, j, k) trace_pt(role, j, k)
#else
#define SSD_TRACE_PT(role, j, k) ((void)0)
#endif

struct TcParams {
    int batch, L, H, nblk, dir, accumulate;
    const __nv_bfloat16 *dt;
    const float *A, *D;
    __nv_bfloat16 *y;
    int *status;
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on phase `parity` by the lanes in `mask` (all of them call it).
// Returns false (after raising the CTA abort flag and the global status word)
// if the phase does not complete in time, or if another thread of the CTA has
// already aborted; the result is the same for every lane in `mask`.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t mask, volatile int *abort_flag,
                                       int *status, int code) {
    bool ok = mbar_try(bar, parity);
    if (!ok) {
        const long long t0 = clock64();
        while (true) {
            if (mbar_try(bar, parity)) { ok = true; break; }
            if (*abort_flag) break;
            if (clock64() - t0 > kWaitCycles) {
                *abort_flag = 1;
                atomicExch(status, code);
                break;
            }
        }
    }
    return __all_sync(mask, ok);
}

// Bounded wait that ignores the abort flag: used on the way out to let
// copies already in flight land before the CTA releases its shared memory.
__device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try(bar, parity) && clock64() - t0 < kWaitCycles) {
    }
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 "version 1").
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: f32 accumulate, bf16 A and B, M = 128.
__host__ __device__ constexpr uint32_t idesc(int n, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
    tmem_st16(taddr, r);
    tmem_st16(taddr + 16, r + 16);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// byte offset of 16-byte chunk q of row r in a [rows][64] bf16 tile with 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int r, int q) { return (uint32_t)(r * 128 + ((q ^ (r & 7)) << 4)); }


// ------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, 1)
k_ssd_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
         const __grid_constant__ CUtensorMap map_c, TcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    float *cs2_s = reinterpret_cast<float *>(sm + kOffCS);          // [2][128] cs * log2(e)
    float *dt_s = cs2_s + 2 * kBlk;                                  // [2][128] dt
    float *red = reinterpret_cast<float *>(sm + kOffRed);            // [2 WG][8]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npairs = prm.H / 2;
    const int b = blockIdx.x / npairs, hp = blockIdx.x % npairs;
    const int h0 = 2 * hp;
    const int nblk = prm.nblk, dir = prm.dir, L = prm.L;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        const uint32_t counts[kNumBars] = {1, 1, 8, 8, 1, 1, 1, 8, 8, 1, 8, 8, 1, 8, 8, 1, 8, 1, 4, 4};
        for (int i = 0; i < (int)kNumBars; ++i) mbar_init(bar(i), counts[i]);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint32_t MASK = 1u;
            int issued = 0;   // blocks whose loads were issued
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_c)) : "memory");
            for (int j = 0; j < nblk; ++j) {
                const int cm = dir > 0 ? j : nblk - 1 - j;
                const int row = b * L + cm * kBlk;
                const int st = j & 1;
                if (j >= 2 && !mbar_wait(bar(B_XEMPTY0 + st), ((j >> 1) - 1) & 1, MASK, abort_flag, prm.status, 11)) break;
                SSD_TRACE_PT(0, j, 0);
                mbar_expect_tx(bar(B_XFULL0 + st), 2 * kTileBytes);
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(sbase + kOffX + (st * 2 + h) * kTileBytes, &map_x, (h0 + h) * kP, row,
                                bar(B_XFULL0 + st));
                if (j >= 1 && !mbar_wait(bar(B_BCEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 12)) break;
                SSD_TRACE_PT(0, j, 1);
                mbar_expect_tx(bar(B_BCFULL), 4 * kTileBytes);
                for (int q = 0; q < 2; ++q) {
                    tma_load_2d(sbase + kOffB + q * kTileBytes, &map_b, q * 64, row, bar(B_BCFULL));
                    tma_load_2d(sbase + kOffC + q * kTileBytes, &map_c, q * 64, row, bar(B_BCFULL));
                }
                issued = j + 1;
            }
            if (*abort_flag && issued > 0) {
                // let copies still in flight land before the CTA exits
                const int j = issued - 1;
                mbar_drain(bar(B_XFULL0 + (j & 1)), (j >> 1) & 1);
                if (j >= 1) mbar_drain(bar(B_XFULL0 + ((j - 1) & 1)), ((j - 1) >> 1) & 1);
                mbar_drain(bar(B_BCFULL), j & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t MASK = 1u;
            const uint32_t id_g = idesc(128, 0, 0), id_s = idesc(128, 1, 1), id_yo = idesc(128, 0, 1),
                           id_yd = idesc(64, 0, 1);
            const uint32_t aB = sbase + kOffB, aC = sbase + kOffC, aWX = sbase + kOffWX, aSP = sbase + kOffSP;
            for (int j = 0; j < nblk; ++j) {
                const int st = j & 1;
                const uint32_t aX = sbase + kOffX + st * 2 * kTileBytes;
                // G = C B^T  (M = rows, N = source rows, K = n)
                if (!mbar_wait(bar(B_BCFULL), j & 1, MASK, abort_flag, prm.status, 21)) break;
                if (j >= 1 && !mbar_wait(bar(B_GEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 22)) break;
                SSD_TRACE_PT(1, j, 0);
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                    mma_ss(tmem + kColG, sdesc(aC + off, 16, 1024), sdesc(aB + off, 16, 1024), id_g, ks > 0);
                }
                mma_commit(bar(B_GFULL));
                // S^T = B^T (w x)  (M = n, N = (head, p), K = rows); both operands MN-major
                if (!mbar_wait(bar(B_WXREADY), j & 1, MASK, abort_flag, prm.status, 23)) break;
                if (j >= 1 && !mbar_wait(bar(B_SEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 24)) break;
                SSD_TRACE_PT(1, j, 1);
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = ks * 2048;
                    mma_ss(tmem + kColS, sdesc(aB + off, kTileBytes, 1024), sdesc(aWX + off, kTileBytes, 1024), id_s,
                           ks > 0);
                }
                mma_commit(bar(B_SFULL));
                // Y = C S'^T of the state entering this block (M = rows, N = (head, p), K = n)
                if (j >= 1) {
                    if (!mbar_wait(bar(B_SPREADY), (j - 1) & 1, MASK, abort_flag, prm.status, 25)) break;
                    if (!mbar_wait(bar(B_YEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 26)) break;
                    SSD_TRACE_PT(1, j, 2);
                    tc_fence_after();
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t offc = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                        mma_ss(tmem + kColY, sdesc(aC + offc, 16, 1024), sdesc(aSP + ks * 2048, kTileBytes, 1024), id_yo,
                               ks > 0);
                    }
                    mma_commit(bar(B_YOFFFULL));
                }
                mma_commit(bar(B_BCEMPTY));
                // Y += M_h X_h  (A from TMEM, B = X_h MN-major, N = 64 per head)
                if (!mbar_wait(bar(B_MREADY), j & 1, MASK, abort_flag, prm.status, 27)) break;
                if (j >= 1 && !mbar_wait(bar(B_RSREADY), (j - 1) & 1, MASK, abort_flag, prm.status, 28)) break;
                if (!mbar_wait(bar(B_XFULL0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 29)) break;
                SSD_TRACE_PT(1, j, 3);
                tc_fence_after();
                for (int h = 0; h < 2; ++h)
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ts(tmem + kColY + 64 * h, tmem + kColM + 64 * h + 8 * ks,
                               sdesc(aX + h * kTileBytes + ks * 2048, kTileBytes, 1024), id_yd, (j >= 1) || (ks > 0));
                mma_commit(bar(B_YFULL));
            }
            // drain: every MMA issued above has completed before TMEM is released
            mma_commit(bar(B_DONE));
            mbar_drain(bar(B_DONE), 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------- per-head CUDA-core work
        const int wg = (warp - 4) >> 2;            // 0: head h0, 1: head h0+1
        const int wq = warp & 3;                   // TMEM lane quarter
        const int r = wq * 32 + lane;              // row in block == TMEM lane
        const int h = h0 + wg;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        const float A2 = prm.A[h] * kLog2e;        // log2 units: exp(a) = exp2(a * log2 e)
        const float Dh = prm.D ? prm.D[h] : 0.f;
        const uint32_t MASK = 0xffffffffu;
        uint32_t wg_phase = 0;   // completions of this WG's sync barrier so far
        // bounded replacement for a named barrier over the 4 warps of this WG
        auto wg_sync = [&](int code) -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_WG0 + wg));
            const bool ok = mbar_wait(bar(B_WG0 + wg), wg_phase & 1, MASK, abort_flag, prm.status, code);
            ++wg_phase;
            return ok;
        };
        {
            // M_h outside the causal triangle is never written: start it at zero
            const uint32_t z[16] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
            for (int c = 0; c < 64; c += 16) tmem_st16(tl + kColM + 64 * wg + c, z);
            tmem_wait_st();
        }
        float state[kP];
#pragma unroll
        for (int i = 0; i < kP; ++i) state[i] = 0.f;
        float *cs2 = cs2_s + wg * kBlk, *dts = dt_s + wg * kBlk;
        uint8_t *wx_tile = sm + kOffWX + wg * kTileBytes;
        uint8_t *sp_tile = sm + kOffSP + wg * kTileBytes;
        auto tok_of = [&](int j) { return (dir > 0 ? j : nblk - 1 - j) * kBlk + r; };
        float dt_next = __bfloat162float(prm.dt[((size_t)b * L + tok_of(0)) * prm.H + h]);

        for (int j = 0; j < nblk; ++j) {
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            const int st = j & 1;
            const int t = tok_of(j);
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 0);
            const float dtr = dt_next;
            if (j + 1 < nblk) dt_next = __bfloat162float(prm.dt[((size_t)b * L + tok_of(j + 1)) * prm.H + h]);

            // cumulative A*dt in scan order (prefix over rows forward, suffix over rows reverse)
            float s = dtr;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = dir > 0 ? __shfl_up_sync(0xffffffffu, s, o) : __shfl_down_sync(0xffffffffu, s, o);
                if (dir > 0 ? lane >= o : lane + o < 32) s += u;
            }
            if (!wg_sync(51)) break;           // previous block's readers of red/cs are done
            if (lane == (dir > 0 ? 31 : 0)) red[wg * 8 + wq] = s;
            if (!wg_sync(52)) break;
            float base = 0.f, total = 0.f;
            for (int w = 0; w < 4; ++w) {
                const float v = red[wg * 8 + w];
                total += v;
                if (dir > 0 ? w < wq : w > wq) base += v;
            }
            const float c2 = A2 * (base + s);                 // cs_r * log2 e
            const float cl2 = A2 * total;                     // cs at the block's last scan position
            cs2[r] = c2;
            dts[r] = dtr;
            const float wr = exp2f(cl2 - c2) * dtr;           // weight of row r in the block's state
            const float er = exp2f(c2);                       // decay from the block start to row r
            const float ablk = exp2f(cl2);                    // decay across the whole block

            // w (.) x -> wX tile (same swizzled layout as the X tile)
            if (!mbar_wait(bar(B_XFULL0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 41)) break;
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 1);
            const uint8_t *xt = sm + kOffX + (st * 2 + wg) * kTileBytes;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 v = *reinterpret_cast<const uint4 *>(xt + swz(r, q));
                uint4 o;
                o.x = pack_bf16(bf16lo(v.x) * wr, bf16hi(v.x) * wr);
                o.y = pack_bf16(bf16lo(v.y) * wr, bf16hi(v.y) * wr);
                o.z = pack_bf16(bf16lo(v.z) * wr, bf16hi(v.z) * wr);
                o.w = pack_bf16(bf16lo(v.w) * wr, bf16hi(v.w) * wr);
                *reinterpret_cast<uint4 *>(wx_tile + swz(r, q)) = o;
            }
            fence_async_smem();
            if (!wg_sync(53)) break;           // cs2/dts of all rows visible to this WG
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 2);
            if (lane == 0) mbar_arrive(bar(B_WXREADY));

            // M_h = G (.) decay (.) dt over the causal triangle, bf16 into TMEM
            if (!mbar_wait(bar(B_GFULL), j & 1, MASK, abort_flag, prm.status, 42)) break;
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 3);
            tc_fence_after();
            for (int kb = 0; kb < 4; ++kb) {
                const bool need = dir > 0 ? kb <= wq : kb >= wq;
                if (!need) continue;           // entirely outside the triangle: stays zero from set-up
                float g[32];
                tmem_ld32(tl + kColG + kb * 32, g);
                tmem_wait_ld();
                uint32_t m[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float mv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int sidx = kb * 32 + 2 * i + e;
                        const bool in = dir > 0 ? sidx <= r : sidx >= r;
                        mv[e] = in ? g[2 * i + e] * exp2f(c2 - cs2[sidx]) * dts[sidx] : 0.f;
                    }
                    m[i] = pack_bf16(mv[0], mv[1]);
                }
                tmem_st16(tl + kColM + 64 * wg + kb * 16, m);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_GEMPTY));
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 10);

            // state: S' <- exp(cs_last) S' + S, thread r holds state row n = r
            if (!mbar_wait(bar(B_SFULL), j & 1, MASK, abort_flag, prm.status, 43)) break;
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 4);
            tc_fence_after();
            {
                float sv[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tl + kColS + 64 * wg + 32 * half, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) state[32 * half + i] = fmaf(ablk, state[32 * half + i], sv[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SEMPTY));
            if (j + 1 < nblk) {
                // the previous state tile must have been consumed by this block's Y = C S'^T
                if (j >= 1 && !mbar_wait(bar(B_YOFFFULL), (j - 1) & 1, MASK, abort_flag, prm.status, 44)) break;
                if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 5);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 o;
                    o.x = pack_bf16(state[8 * q + 0], state[8 * q + 1]);
                    o.y = pack_bf16(state[8 * q + 2], state[8 * q + 3]);
                    o.z = pack_bf16(state[8 * q + 4], state[8 * q + 5]);
                    o.w = pack_bf16(state[8 * q + 6], state[8 * q + 7]);
                    *reinterpret_cast<uint4 *>(sp_tile + swz(r, q)) = o;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SPREADY));
            }

            // Y (from the incoming state) scaled by exp(cs_r), before the intra-block term is added
            if (j >= 1) {
                if (!mbar_wait(bar(B_YOFFFULL), (j - 1) & 1, MASK, abort_flag, prm.status, 45)) break;
                if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 6);
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float yv[32];
                    tmem_ld32(tl + kColY + 64 * wg + 32 * half, yv);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) yv[i] *= er;
                    tmem_st32(tl + kColY + 64 * wg + 32 * half, yv);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_RSREADY));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_MREADY));

            // epilogue: y = Y + D x, bf16, 128 contiguous bytes per thread
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 7);
            if (!mbar_wait(bar(B_YFULL), j & 1, MASK, abort_flag, prm.status, 46)) break;
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 8);
            tc_fence_after();
            float yv[64];
            tmem_ld32(tl + kColY + 64 * wg, yv);
            tmem_ld32(tl + kColY + 64 * wg + 32, yv + 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_YEMPTY));
            __nv_bfloat16 *yrow = prm.y + (((size_t)b * L + t) * prm.H + h) * kP;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xt + swz(r, q));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                float o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[2 * i] = fmaf(Dh, bf16lo(xw[i]), yv[8 * q + 2 * i]);
                    o[2 * i + 1] = fmaf(Dh, bf16hi(xw[i]), yv[8 * q + 2 * i + 1]);
                }
                if (prm.accumulate) {
                    const uint4 pv = *reinterpret_cast<const uint4 *>(yrow + 8 * q);
                    const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        o[2 * i] += bf16lo(pw[i]);
                        o[2 * i + 1] += bf16hi(pw[i]);
                    }
                }
                uint4 ov;
                ov.x = pack_bf16(o[0], o[1]);
                ov.y = pack_bf16(o[2], o[3]);
                ov.z = pack_bf16(o[4], o[5]);
                ov.w = pack_bf16(o[6], o[7]);
                *reinterpret_cast<uint4 *>(yrow + 8 * q) = ov;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_XEMPTY0 + st));
            if (warp == 4 && lane == 0) SSD_TRACE_PT(2, j, 9);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encode() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// [rows][cols] bf16 matrix, row-major; box [128 rows][64 cols], 128-byte swizzle
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kBlk};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(bool bf16, int batch, int L, int H, int P, int N, int G, int chunk) {
    (void)batch;
    return bf16 && P == kP && N == kN && G == 1 && H % 2 == 0 && chunk % kBlk == 0 && L % kBlk == 0 &&
           (long long)batch * L <= (1ll << 31) - 1 && get_encode() != nullptr;
}

size_t tc_workspace_bytes(int, int, int, int) { return 0; }

TcArgs make_tc_args(int batch, int L, int H, int chunk, void *ws, int *status) {
    TcArgs t{};
    t.batch = batch; t.L = L; t.H = H; t.chunk = chunk; t.ws = ws; t.status = status;
    return t;
}

void tc_set_direction(TcArgs &t, int slot, int dir, const void *x, const void *dt, const float *A, const void *B,
                      const void *C, const float *D) {
    t.d[slot] = TcDir{x, dt, B, C, A, D, dir};
}

int tc_launches(bool bidir) { return bidir ? 2 : 1; }

#ifdef SSD_TRACE
extern "C" int ssd_debug_trace(unsigned long long *out, int n) {
    const int total = 3 * kTraceBlocks * kTracePts;
    if (n < total) return -1;
    return cudaMemcpyFromSymbol(out, g_trace, sizeof(unsigned long long) * total) == cudaSuccess ? total : -2;
}
#endif

cudaError_t launch_tc(const TcArgs &t, bool bidir, void *y, cudaStream_t st) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(k_ssd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int ndir = bidir ? 2 : 1;
    for (int s = 0; s < ndir; ++s) {
        const TcDir &d = t.d[s];
        CUtensorMap mx, mb, mc;
        const uint64_t rows = (uint64_t)t.batch * t.L;
        if (!make_map(&mx, d.x, rows, (uint64_t)t.H * kP) || !make_map(&mb, d.B, rows, kN) ||
            !make_map(&mc, d.C, rows, kN))
            return cudaErrorInvalidValue;
        TcParams p{};
        p.batch = t.batch; p.L = t.L; p.H = t.H; p.nblk = t.L / kBlk; p.dir = d.dir; p.accumulate = s;
        p.dt = static_cast<const __nv_bfloat16 *>(d.dt);
        p.A = d.A; p.D = d.D;
        p.y = static_cast<__nv_bfloat16 *>(y);
        p.status = t.status;
        k_ssd_tc<<<t.batch * (t.H / 2), kThreads, kSmemBytes, st>>>(mx, mb, mc, p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ssd
