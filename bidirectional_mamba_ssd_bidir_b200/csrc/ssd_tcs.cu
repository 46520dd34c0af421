// ssd_tcs.cu -- tensor-core (tcgen05 / TMEM / TMA) SSD scan for bf16 io,
// headdim 64, d_state 128, one B/C group, with the masked score matrix shared
// by the two heads of a CTA.
//
// This is the chunked evaluation of the recurrence S <- exp(dt A) S +
// dt x (outer) B, y = C.S + D x that the Mamba-2 layers of the DiffuMamba
// mixer ("DiffuMamba", technical summary, section 2: two independent layers,
// forward and reverse) and the R2LM right-to-left stream ("Bifocal Diffusion
// Language Models", section 2, mechanism: flip, scan, flip back) run.  The
// reverse direction is the forward algebra in scan order with every token
// index mapped t -> L-1-t in the address arithmetic only.
//
// One CTA owns (batch b, head pair {h0, h0+1}, direction) and walks the
// sequence in scan order in blocks of 128 tokens.  In scan positions k of one
// block, with cs_k = A_h * (dt_0 + ... + dt_k) (inclusive, <= 0, decreasing):
//
//   y_k = sum_{i<=k} (C_k.B_i) exp(cs_k - cs_i) dt_i x_i + exp(cs_k) C_k.S_in + D x_k
//   S_out = exp(cs_127) S_in + sum_i exp(cs_127 - cs_i) dt_i x_i (outer) B_i
//
// The decay splits around the block's mid-point m = (cs_0 + cs_127) / 2:
// exp(cs_k - cs_i) = r_k c_i / dt_i with r_k = exp(cs_k - m) and
// c_i = exp(m - cs_i) dt_i, both within 2^(+-D/2) for a block decay D.  So
//
//   y_k = r_k [ (Gc (cX))_k + C_k.(e^m S_in) ] + D x_k,   Gc = (C B^T) masked to i <= k,
//   S_out = kappa [ e^m S_in + B^T (cX) ],                kappa = exp(cs_127 - m),
//
// where cX = c (.) X scales the rows of the x tile.  Gc does not depend on the
// head (one B/C group), so it is formed once per block for both heads, on the
// tensor core and masked once; the per-head decay lives only in the row factor
// r (epilogue), in the row scaling of x (which the state product shares), and
// in two scalars per head and block.  Per block, on the tensor core:
//
//   G    = C B^T                          TMEM [0,128), two N = 64 halves
//   Y_j  = D x / r                        CUDA cores (tcgen05.st), Y buffer j & 1
//   Y_j += C (e^m S_in)^T                 A = C, B = bf16 copy of the scaled state (smem)
//   S   <- e^m S_in (scaled in place);    S += B^T (cX)     TMEM [128,256)
//   Y_j += Gc (cX)                        A = Gc (bf16, in place over G), B = cX
//   y    = r Y_j                          CUDA cores -> smem (the B buffer) -> TMA store
//
// A block whose decay D exceeds 2^kSteepLog2 would push r or c out of float
// range; a CTA whose chain has such a block runs nothing here and the exact
// kernel (ssd_tc.cu) runs it afterwards (see launch_tc).
//
// Bidirectional mixer in one launch: the CTAs of the forward and reverse
// scans of a head pair are neighbours in the grid.  For every output block of
// the head pair, an epoch-tagged ticket makes one direction first: it stores
// its part of y and publishes an epoch-tagged ready word; the other, second,
// adds its part once that word is published, with a TMA bf16 reduce-add
// (performed in L2).  The first never waits, so the hand-off cannot deadlock
// whatever the residency.
//
// Warp roles (640 threads): warps 0-15 are the CUDA-core warps (warp w: TMEM
// lane quarter w & 3, column group w >> 2 of 32 columns; the head of a column
// group is (w >> 2) >> 1); warp 16 issues the x, C and dt loads and builds the
// decay tables; warps 17 and 19 issue the MMAs, two independent streams (17
// also owns TMEM); warp 18
// takes the forward/reverse tickets, stores y (TMA), publishes first parts and
// loads B into each buffer as soon as its y tile has been read.  The CUDA-core
// warps never wait for global memory or for the other direction.  Every wait is
// bounded; a wait that runs out records SSD_ERR_TIMEOUT in the status word and
// the CTA winds down without touching more data.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstring>

#include "ssd_tc.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kBlk = 128;            // tokens per block (MMA M)
constexpr int kP = 64, kN = 128;
constexpr int kThreads = 640;
constexpr int kWarpLoad = 16, kWarpMmaA = 17, kWarpStore = 18, kWarpMmaB = 19;
constexpr uint32_t kTileBytes = kBlk * 64 * 2;        // one [128][64] bf16 swizzled tile = 16 KB
constexpr uint32_t kPairBytes = 2 * kTileBytes;       // two tiles (two heads, or two 64-column halves)
constexpr uint32_t kDtBytes = kBlk * 8 * 2;           // dt box: 128 tokens x 8 heads, bf16

// TMEM columns: G (Gc over it), the state, two Y accumulators
constexpr uint32_t kColG = 0, kColS = 128, kColY = 256;

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t kOffX = 0;                           // 2 stages: x, scaled in place to cX
constexpr uint32_t kOffB = kOffX + 2 * kPairBytes;      // 2 buffers: B (n halves), then the y tile (heads)
constexpr uint32_t kOffC = kOffB + 2 * kPairBytes;      // C (n halves)
constexpr uint32_t kOffS = kOffC + kPairBytes;          // bf16 scaled state, rows = n, one tile per head
constexpr uint32_t kOffTab = kOffS + kPairBytes;        // 3 table buffers (block j in buffer j % 3)
// one table buffer (floats): row factor r, column factor c = e dt, prestore factor e D (per head
// and row, memory order), and per head the mid-point m and kappa exponent (log2 units)
constexpr uint32_t kTabR = 0, kTabCF = 2 * kBlk, kTabDR = 4 * kBlk, kTabM2 = 6 * kBlk, kTabK2 = 6 * kBlk + 2;
constexpr uint32_t kTabFloats = 6 * kBlk + 8;
constexpr uint32_t kOffDT = (kOffTab + 3 * kTabFloats * 4 + 127) / 128 * 128;   // dt ring, 3 slots
constexpr uint32_t kOffBar = kOffDT + 3 * kDtBytes;

enum Bar {
    B_XFULL0 = 0, B_XFULL1, B_XEMPTY0, B_XEMPTY1, B_BFULL0, B_BFULL1, B_CFULL, B_CEMPTY,
    B_DTFULL0, B_DTFULL1, B_DTFULL2, B_GFULL, B_GCREADY, B_CXREADY0,
    B_CXREADY1, B_STFULL, B_SREADY, B_YOFFDONE, B_YFULL, B_TABREADY0, B_TABREADY1, B_TABREADY2,
    B_TABFREE0, B_TABFREE1, B_TABFREE2, B_TILE0, B_TILE1, B_DONEA, B_DONEB, kNumBars
};
// misc: tmem base, abort flag, wait limit
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 32 + 1024;   // + alignment slack
static_assert(kPairBytes % 1024 == 0, "tiles must stay 1024-byte aligned");
static_assert(kOffBar % 8 == 0 && kOffMisc % 8 == 0, "barrier alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr float kLog2e = 1.4426950408889634f;
// a block whose decay passes this (log2 units) is outside what the steep test admits: the
// factors would leave float range; the CTA aborts with a status code instead
constexpr float kGuardLog2 = 240.f;

// Optional phase timeline for the tracing build (-DSSD_TRACE): SM-clock stamps
// of CTA 0, first kTraceBlocks blocks, per warp and phase; and every CTA's
// start and end on the global timer, with its SM.
#ifdef SSD_TRACE
constexpr int kTraceWarps = 20, kTraceBlocks = 8, kTracePts = 24;
__device__ unsigned long long g_trace[kTraceWarps][kTraceBlocks][kTracePts];
__device__ __forceinline__ void trace_pt(int w, int j, int k) {
    if (blockIdx.x == 0 && j >= 0 && j < kTraceBlocks && (threadIdx.x & 31) == 0) {
        g_trace[w][j][k] = (unsigned long long)clock64();   // SM cycles: exact within the CTA
    }
}
#define SSD_TRACE_PT(w, j, k) trace_pt(w, j, k)
// per-block timeline of CTAs 0 and 1 (the two directions of the first head pair), every block:
// 0 G issued, 1 y store issued, 2 y tiles read (B buffer free), 3 B load issued
constexpr int kTraceAllBlocks = 1024;
__device__ unsigned long long g_blk[2][kTraceAllBlocks][4];
#define SSD_TRACE_BLK(j, k)                                                                   \
    do {                                                                                      \
        if (blockIdx.x < 2 && (j) < kTraceAllBlocks && (threadIdx.x & 31) == 0)               \
            g_blk[blockIdx.x][j][k] = (unsigned long long)clock64();                          \
    } while (0)
__device__ unsigned long long g_cta_time[4096][3];     // start, end, SM id
#define SSD_TRACE_CTA(k)                                                              \
    do {                                                                              \
        if (threadIdx.x == 0 && blockIdx.x < 4096) {                                  \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                    \
            g_cta_time[blockIdx.x][k] = t_;                                           \
            unsigned smid_;                                                           \
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));                        \
            g_cta_time[blockIdx.x][2] = smid_;                                        \
        }                                                                             \
    } while (0)
#else
#define SSD_TRACE_CTA(k) ((void)0)
#define SSD_TRACE_PT(w, j, k) ((void)0)
#define SSD_TRACE_BLK(j, k) ((void)0)
#endif

struct TcsDirParams {
    const float *A, *D;
    const __nv_bfloat16 *dt;
};

struct TcsParams {
    int batch, L, H, nblk;
    __nv_bfloat16 *y;
    int bidir;                          // 1: slot = blockIdx & 1, forward/reverse hand-off through flags
    int dir_single;                     // direction of slot 0 when bidir == 0
    TcsDirParams d[2];
    int *status;
    unsigned long long *ticket;         // [batch][H][nblk], epoch-tagged (bidir only)
    unsigned long long *ready;          // [batch][H][nblk], epoch-tagged (bidir only)
    unsigned long long epoch;
    long long wait_cycles;              // bound of every device-side wait
    int fault;                          // test hook: 1 = the first direction never publishes its part
    const float *s_in;                  // single direction: [batch][H][P][N] state entering the scan, or null
    float *s_out;                       // single direction: [batch][H][P][N] state leaving the scan, or null
    // sequence segments (nseg > 1): a CTA runs sb blocks of its chain; the state entering its
    // segment folds the local end states of the pieces (npiece per segment) before it
    int nseg, sb, npiece;
    const float *sloc;                  // [batch][H][2][(nseg - 1) npiece][P][N]
    const float *ldec;                  // [batch][H][2][(nseg - 1) npiece]: A * (sum of dt), log2 units
    const unsigned long long *steep;    // [batch][H/2][2], epoch-tagged: chains left to the exact kernel
};

struct TcsMaps {
    CUtensorMap x[2], dt[2], b[2], c[2], y;
};

__global__ void __launch_bounds__(kThreads, 1) k_ssd_tcs(const __grid_constant__ TcsMaps maps,
                                                         const __grid_constant__ TcsParams prm) {
    // Dependents launched programmatically behind this grid (the exact kernel for the steep
    // chains) may start as soon as every CTA of it has started.
    asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);   // limit at +8
    float *tab_s = reinterpret_cast<float *>(sm + kOffTab);         // [3 buffers][kTabFloats]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npairs = prm.H / 2;
    const int unit = prm.bidir ? (blockIdx.x >> 1) : blockIdx.x;
    const int slot = prm.bidir ? (blockIdx.x & 1) : 0;
    const int dir = prm.bidir ? (slot == 0 ? 1 : -1) : prm.dir_single;
    const int seg = unit % prm.nseg, pu = unit / prm.nseg;
    const int b = pu / npairs, hp = pu % npairs;
    const int h0 = 2 * hp;
    const int nblk_chain = prm.nblk, L = prm.L;
    // this CTA's blocks: scan-order blocks g0 .. g0 + nblk - 1 of the chain
    const int g0 = seg * prm.sb;
    const int nblk = min(prm.sb, nblk_chain - g0);
    const CUtensorMap *map_x = &maps.x[slot], *map_dt = &maps.dt[slot], *map_b = &maps.b[slot],
                      *map_c = &maps.c[slot];
    // a state enters this CTA's blocks: the caller's (single direction), or a segment's before it
    const int has_in = prm.s_in != nullptr || seg > 0;
    float *const s_out = seg == prm.nseg - 1 ? prm.s_out : nullptr;   // left by the chain's last segment

    // A chain with a block too steep for the factorised decay is left to the exact kernel: the
    // call's steep marks (made by the state kernel when segmented, by one pass otherwise) say which.
    const bool steep =
        *reinterpret_cast<const volatile unsigned long long *>(prm.steep + ((size_t)b * npairs + hp) * 2 + slot) ==
        prm.epoch;
    if (nblk <= 0) return;
    if (steep) return;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < (int)kNumBars; ++i) {
            // arrivals: 16 = one per CUDA-core warp, 1 = one thread or one MMA commit (TMA
            // completions count bytes)
            uint32_t cnt = 1;
            if (i == B_GCREADY || i == B_CXREADY0 || i == B_CXREADY1 || i == B_SREADY) cnt = 16;
            if (i == B_TILE0 || i == B_TILE1 || (i >= B_TABFREE0 && i <= B_TABFREE2)) cnt = 16;
            // read by both MMA streams: a commit from each
            if (i == B_XEMPTY0 || i == B_XEMPTY1 || i == B_CEMPTY) cnt = 2;
            mbar_init(bar(i), cnt);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMmaA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    SSD_TRACE_CTA(0);

    // memory block of this CTA's block jj, and its first token row
    auto mblk_of = [&](int jj) { return dir > 0 ? g0 + jj : nblk_chain - 1 - (g0 + jj); };
    auto row_of = [&](int jj) { return b * L + mblk_of(jj) * kBlk; };
    if (warp == kWarpLoad) {
        // ---------------------------------------------------------- TMA loads, tables
        // Lane 0 issues the loads as their buffers free up: x of block j once block j-2's
        // products have read its stage, C once block j-1's products have read it, dt three
        // blocks ahead of the tables.  (B is loaded by the store warp, into the buffer its y
        // store has just read.)  No L2 prefetches: measured, they cost more copy-engine time
        // than they save in load latency.
        // The whole warp builds the decay tables (the CUDA-core warps never compute them).
        const uint32_t MASK = 0xffffffffu;
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_x)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_dt)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_b)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_c)) : "memory");
        }
        int x_issued = 0, c_issued = 0, dt_issued = 0;
        // dt of block jj into slot jj % 3, loaded once the tables of block jj-3 (the slot's
        // previous content) have been built, in this warp's program order
        auto load_dt = [&](int jj) {
            const int sl = jj % 3;
            if (lane == 0) {
                mbar_expect_tx(bar(B_DTFULL0 + sl), kDtBytes);
                tma_load_2d(sbase + kOffDT + sl * kDtBytes, map_dt, h0 & ~7, row_of(jj), bar(B_DTFULL0 + sl));
            }
            dt_issued = jj + 1;
        };
        // Tables of block jj (buffer jj % 3), both heads: lane l takes scan positions 4l..4l+3
        // (memory rows k forward, 127 - k reverse), forms the inclusive cumulative A dt in scan
        // order (its own four, then a warp scan), the block's mid-point m and the factors.
        auto build_tables = [&](int jj) -> bool {
            const int sl = jj % 3;
            if (!mbar_wait(bar(B_DTFULL0 + sl), (jj / 3) & 1, MASK, abort_flag, prm.status, 51)) return false;
            const uint8_t *dtt = sm + kOffDT + sl * kDtBytes;      // [128 rows][8 heads] bf16
            float *tb = tab_s + (jj % 3) * kTabFloats;
            const int hc = h0 & 7;                                  // column of head h0 (h0 + 1 next to it)
            int rows[4];
            uint32_t dpair[4];                                      // (head h0, head h0 + 1) dt of each row
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int k = 4 * lane + i;
                rows[i] = dir > 0 ? k : kBlk - 1 - k;
                dpair[i] = *reinterpret_cast<const uint32_t *>(dtt + rows[i] * 16 + hc * 2);
            }
            bool ok = true;
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                float d[4], p[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) d[i] = hs ? bf16hi(dpair[i]) : bf16lo(dpair[i]);
                p[0] = d[0]; p[1] = p[0] + d[1]; p[2] = p[1] + d[2]; p[3] = p[2] + d[3];
                float incl = p[3];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(MASK, incl, o);
                    if (lane >= o) incl += u;
                }
                const float excl = incl - p[3];
                const float total = __shfl_sync(MASK, incl, 31), dfirst = __shfl_sync(MASK, d[0], 0);
                const float A2 = prm.d[slot].A[h0 + hs] * kLog2e;
                const float Dh = prm.d[slot].D ? prm.d[slot].D[h0 + hs] : 0.f;
                const float cf2 = A2 * dfirst, cl2 = A2 * total;   // cs at the first and last scan positions
                const float m2 = 0.5f * (cf2 + cl2);
                // outside what the steep test admits (it cannot happen for a chain that passed it)
                if (!(cf2 - cl2 <= kGuardLog2)) ok = false;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float cs2 = A2 * (excl + p[i]);
                    const float e = ex2_ftz(m2 - cs2);
                    tb[kTabR + hs * kBlk + rows[i]] = ex2_ftz(cs2 - m2);
                    tb[kTabCF + hs * kBlk + rows[i]] = e * d[i];
                    tb[kTabDR + hs * kBlk + rows[i]] = e * Dh;
                }
                if (lane == 0) {
                    tb[kTabM2 + hs] = m2;
                    tb[kTabK2 + hs] = cl2 - m2;
                }
            }
            if (!ok) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(prm.status, 71);
                }
                return false;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_TABREADY0 + jj % 3));
            return true;
        };
        // Three independent in-order streams, served by readiness (C first: it gates the next
        // block's scores; then x, the tables with dt).  Each buffer's wait condition is a parity
        // test on a barrier that is at most one phase away from the awaited one, since its
        // stream issues in block order.
        for (int jj = 0; jj < 3 && jj < nblk; ++jj) load_dt(jj);
        int tb_built = 0;
        long long t_idle = clock64();
        const long long limit = *reinterpret_cast<volatile long long *>(abort_flag + 1);
        while (c_issued < nblk || x_issued < nblk || tb_built < nblk) {
            if (*abort_flag) break;
            uint32_t ready = 0;
            if (lane == 0) {
                if (c_issued < nblk && (c_issued == 0 || mbar_test(bar(B_CEMPTY), (c_issued - 1) & 1)))
                    ready |= 1u;
                if (x_issued < nblk &&
                    (x_issued < 2 || mbar_test(bar(B_XEMPTY0 + (x_issued & 1)), ((x_issued >> 1) - 1) & 1)))
                    ready |= 4u;
                // tables of block t go to buffer t % 3, free once every CUDA-core warp has read
                // block t-3's tables for the last time (its epilogue, B_TABFREE)
                if (tb_built < nblk &&
                    (tb_built < 3 || mbar_test(bar(B_TABFREE0 + tb_built % 3), ((tb_built - 3) / 3) & 1)) &&
                    mbar_test(bar(B_DTFULL0 + tb_built % 3), (tb_built / 3) & 1))
                    ready |= 8u;
            }
            ready = __shfl_sync(MASK, ready, 0);
            if (ready & 1u) {
                const int j = c_issued;
                SSD_TRACE_PT(kWarpLoad, j, 2);
                if (lane == 0) {
                    mbar_expect_tx(bar(B_CFULL), kPairBytes);
                    for (int q = 0; q < 2; ++q)
                        tma_load_2d(sbase + kOffC + q * kTileBytes, map_c, q * 64, row_of(j), bar(B_CFULL));
                }
                c_issued = j + 1;
            }
            if (ready & 4u) {
                const int j = x_issued, sx = j & 1;
                SSD_TRACE_PT(kWarpLoad, j, 0);
                if (lane == 0) {
                    mbar_expect_tx(bar(B_XFULL0 + sx), kPairBytes);
                    // x is read by this CTA only: first out of L2 (B, C and dt are shared by the
                    // head pairs of a batch row and keep the default priority)
                    const uint64_t pol = l2_evict_first();
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_hint(sbase + kOffX + sx * kPairBytes + h * kTileBytes, map_x, (h0 + h) * kP,
                                         row_of(j), bar(B_XFULL0 + sx), pol);
                }
                x_issued = j + 1;
            }
            if (ready & 8u) {
                if (!build_tables(tb_built)) break;
                SSD_TRACE_PT(kWarpLoad, tb_built, 3);
                ++tb_built;
                // dt slot (t + 3) % 3 held the block whose tables were just built
                if (dt_issued < nblk) load_dt(dt_issued);
            }
            if (ready) {
                t_idle = clock64();
            } else if (clock64() - t_idle > limit) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(prm.status, 13);
                }
                break;
            } else {
                __nanosleep(32);
            }
        }
        __syncwarp();
        if (*abort_flag && lane == 0) {
            // let copies still in flight land before the CTA exits
            for (int jj = x_issued - 1; jj >= 0 && jj >= x_issued - 2; --jj)
                mbar_drain(bar(B_XFULL0 + (jj & 1)), (jj >> 1) & 1, prm.wait_cycles);
            if (c_issued > 0) mbar_drain(bar(B_CFULL), (c_issued - 1) & 1, prm.wait_cycles);
            for (int jj = dt_issued - 1; jj >= 0 && jj >= dt_issued - 3; --jj)
                mbar_drain(bar(B_DTFULL0 + jj % 3), (jj / 3) & 1, prm.wait_cycles);
        }
        __syncwarp();
    } else if (warp == kWarpMmaA || warp == kWarpMmaB) {
        // ---------------------------------------------------------- MMA issue, two streams
        // Issuing an MMA costs its thread about as long as an N = 128 product runs, and more
        // while the CUDA-core warps are busy, so one thread cannot keep the tensor core fed.
        // Two warps on different SM sub-partitions issue, each into accumulators of its own:
        //   stream A (warp 17): G = C B^T, then S += B^T (cX)        (TMEM [0,256))
        //   stream B (warp 19): Y_off = C (e^m S_in)^T, then Y_diag   (the Y buffers)
        // Whole warps run the loops; one elected lane issues.  Between the streams: G of the
        // next block waits for this block's Y_diag (Gc lies over G); the bf16 state copy read by
        // Y_off is rewritten only after Y_off (B_YOFFDONE); buffers both streams read free on a
        // commit from each.
        const uint32_t MASK = 0xffffffffu;
        const bool stream_a = warp == kWarpMmaA;
        const uint32_t id_g = idesc(128, 0, 0),          // G: M = rows, N = sources, K = n
            id_s = idesc(128, 1, 1),                      // state: M = n, N = (head, p), K = rows
            id_y = idesc(128, 0, 1);                      // Y: M = rows, N = (head, p)
        // operand descriptors, built once: C and B K-major for G and Y_off (rows of 128 bytes,
        // 8-row groups 1 KB apart), B, cX and the state copy MN-major (64-element chunks 16 KB
        // apart, 8-row groups 1 KB apart)
        const SDesc dC = make_sdesc(sbase + kOffC, 16, 1024), dS = make_sdesc(sbase + kOffS, kTileBytes, 1024);
        const SDesc dBk0 = make_sdesc(sbase + kOffB, 16, 1024), dBk1 = make_sdesc(sbase + kOffB + kPairBytes, 16, 1024);
        const SDesc dBm0 = make_sdesc(sbase + kOffB, kTileBytes, 1024),
                    dBm1 = make_sdesc(sbase + kOffB + kPairBytes, kTileBytes, 1024);
        const SDesc dX0 = make_sdesc(sbase + kOffX, kTileBytes, 1024),
                    dX1 = make_sdesc(sbase + kOffX + kPairBytes, kTileBytes, 1024);
        for (int j = 0; j < nblk; ++j) {
            const int st = j & 1;
            const SDesc dBk = st ? dBk1 : dBk0, dBm = st ? dBm1 : dBm0, dX = st ? dX1 : dX0;
            if (stream_a) {
                if (!mbar_wait(bar(B_BFULL0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 21)) break;
                if (!mbar_wait(bar(B_CFULL), j & 1, MASK, abort_flag, prm.status, 22)) break;
                // G over the columns where the previous block's Gc lies: after its Y_diag
                if (j >= 1 && !mbar_wait(bar(B_YFULL), (j - 1) & 1, MASK, abort_flag, prm.status, 24)) break;
                SSD_TRACE_PT(kWarpMmaA, j, 4);
                tc_fence_after();
                #pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                    mma_ss_w(tmem + kColG, dC.at(off), dBk.at(off), id_g, ks > 0);
                }
                mma_commit_w(bar(B_GFULL));
                mma_commit_w(bar(B_CEMPTY));
                SSD_TRACE_PT(kWarpMmaA, j, 0);
                SSD_TRACE_BLK(j, 0);
                // S (+)= B^T (cX): M = n, N = (head, p), K = rows; both operands MN-major.  The
                // state was scaled in place for this block (B_SREADY); cX is ready (B_CXREADY).
                if (!mbar_wait(bar(B_CXREADY0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 25)) break;
                if ((j >= 1 || has_in) &&
                    !mbar_wait(bar(B_SREADY), (j - 1 + has_in) & 1, MASK, abort_flag, prm.status, 26))
                    break;
                tc_fence_after();
                #pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ss_w(tmem + kColS, dBm.at(ks * 2048), dX.at(ks * 2048), id_s, (j > 0) || has_in || (ks > 0));
                mma_commit_w(bar(B_STFULL));
                mma_commit_w(bar(B_XEMPTY0 + st));
                SSD_TRACE_PT(kWarpMmaA, j, 2);
            } else {
                const uint32_t colY = kColY + 128u * st;
                if (!mbar_wait(bar(B_CFULL), j & 1, MASK, abort_flag, prm.status, 31)) break;
                // Y_j starts at D x / r, stored by the CUDA-core warps with the cX tile
                if (!mbar_wait(bar(B_CXREADY0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 32)) break;
                if (j >= 1 || has_in) {
                    // Y_j += C (e^m S_in)^T; the bf16 copy of the scaled state is in smem
                    if (!mbar_wait(bar(B_SREADY), (j - 1 + has_in) & 1, MASK, abort_flag, prm.status, 33)) break;
                    tc_fence_after();
                    #pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t offc = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                        mma_ss_w(tmem + colY, dC.at(offc), dS.at(ks * 2048), id_y, 1);
                    }
                }
                mma_commit_w(bar(B_CEMPTY));
                mma_commit_w(bar(B_YOFFDONE));
                SSD_TRACE_PT(kWarpMmaB, j, 1);
                // Y_j += Gc (cX): A = Gc from TMEM (K-step ks at column 16 ks), B = cX (both heads)
                if (!mbar_wait(bar(B_GCREADY), j & 1, MASK, abort_flag, prm.status, 34)) break;
                tc_fence_after();
                #pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts_w(tmem + colY, tmem + kColG + 16 * ks, dX.at(ks * 2048), id_y, 1);
                mma_commit_w(bar(B_YFULL));
                mma_commit_w(bar(B_XEMPTY0 + st));
                SSD_TRACE_PT(kWarpMmaB, j, 3);
            }
        }
        // drain: every MMA this stream issued has completed before TMEM is released
        const uint32_t done = bar(stream_a ? B_DONEA : B_DONEB);
        mma_commit_w(done);
        if (lane == 0) mbar_drain(done, 0, prm.wait_cycles);
        __syncwarp();
    } else if (warp == kWarpStore) {
        // ---------------------------------------------------------- tickets, y stores, B loads
        // Per block (scan order): take the head pair's ticket; if the other direction took it
        // first, wait until its part is published.  Then, once the CUDA-core warps have written
        // both heads' y tiles into the block's B buffer: first direction, TMA store; second,
        // TMA bf16 reduce-add (in L2) onto the published part.  As soon as the tiles have been
        // read, B of block j+2 is loaded into the buffer.  A first part is published once its
        // writes have completed, at the start of the next block's turn (before that block's
        // tiles are ready, so the fence and the release cost the store nothing); before this
        // direction waits on a block the other direction took, it publishes what it has
        // pending.  So a publication depends on nothing the other direction still has to do,
        // and the two cannot wait on each other.  One ticket covers both heads.
        if (lane == 0) {
            const uint32_t MASK = 1u;
            int b_issued = 0;
            auto load_b = [&](int jj) {
                const int sb = jj & 1;
                SSD_TRACE_PT(kWarpLoad, jj, 1);
                SSD_TRACE_BLK(jj, 3);
                mbar_expect_tx(bar(B_BFULL0 + sb), kPairBytes);
                for (int q = 0; q < 2; ++q)
                    tma_load_2d(sbase + kOffB + sb * kPairBytes + q * kTileBytes, map_b, q * 64, row_of(jj),
                                bar(B_BFULL0 + sb));
                b_issued = jj + 1;
            };
            int pend = -1;                  // block stored first whose part is not yet published
            size_t pend_slot = 0;
            auto publish = [&]() {          // call once the block's writes have completed
                asm volatile("fence.proxy.async.global;" ::: "memory");
                if (prm.fault != 1) st_release(prm.ready + pend_slot, prm.epoch);
                SSD_TRACE_PT(kWarpStore, pend, 1);
                pend = -1;
            };
            for (int jj = 0; jj < 2 && jj < nblk; ++jj) load_b(jj);
            bool ok = true;
            for (int j = 0; j < nblk && ok; ++j) {
                const int st = j & 1;
                const int cm = mblk_of(j);
                const size_t pair_slot = ((size_t)b * prm.H + h0) * nblk_chain + cm;
                int sec = 0;
                SSD_TRACE_PT(kWarpStore, j, 3);
                if (prm.bidir) {
                    sec = atomicExch(prm.ticket + pair_slot, prm.epoch) == prm.epoch;
                    SSD_TRACE_PT(kWarpStore, j, 4);
                    if (sec) {
                        if (pend >= 0) {
                            bulk_wait0();
                            publish();
                        }
                        const unsigned long long *rp = prm.ready + pair_slot;
                        const long long t0 = clock64();
                        while (ld_acquire(rp) != prm.epoch) {
                            if (*abort_flag) { ok = false; break; }
                            if (clock64() - t0 > prm.wait_cycles) {
                                *abort_flag = 1;
                                atomicExch(prm.status, 47);
                                ok = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                        if (!ok) break;
                    }
                }
                if (pend >= 0) {
                    // the previous block's first part, while the CUDA-core warps still write this
                    // block's tiles: its store has completed by now or soon
                    bulk_wait0();
                    SSD_TRACE_PT(kWarpStore, j, 5);
                    publish();
                }
                if (!mbar_wait(bar(B_TILE0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 61)) break;
                SSD_TRACE_PT(kWarpStore, j, 0);
                SSD_TRACE_BLK(j, 1);
                const uint32_t tile = sbase + kOffB + st * kPairBytes;
                if (!sec) {
                    if (prm.bidir) {
                        // the other direction adds its part to this one later: keep it in L2
                        const uint64_t pol = l2_evict_last();
                        for (int hs = 0; hs < 2; ++hs)
                            tma_store_2d_hint(&maps.y, tile + hs * kTileBytes, (h0 + hs) * kP, b * L + cm * kBlk,
                                              pol);
                    } else {
                        for (int hs = 0; hs < 2; ++hs)
                            tma_store_2d(&maps.y, tile + hs * kTileBytes, (h0 + hs) * kP, b * L + cm * kBlk);
                    }
                } else {
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    const uint64_t pol = l2_evict_first();   // the finished sum
                    for (int hs = 0; hs < 2; ++hs)
                        tma_reduce_add_2d_hint(&maps.y, tile + hs * kTileBytes, (h0 + hs) * kP, b * L + cm * kBlk,
                                               pol);
                }
                bulk_commit();
                bulk_wait_read0();                        // the tiles may be overwritten from here on
                SSD_TRACE_PT(kWarpStore, j, 2);
                SSD_TRACE_BLK(j, 2);
                if (j + 2 < nblk) load_b(j + 2);
                if (prm.bidir && !sec) {
                    pend = j;
                    pend_slot = pair_slot;
                }
            }
            bulk_wait0();                                 // every store has landed before the CTA exits
            if (ok && pend >= 0 && !*abort_flag) publish();
            if (*abort_flag) {
                for (int jj = b_issued - 1; jj >= 0 && jj >= b_issued - 2; --jj)
                    mbar_drain(bar(B_BFULL0 + (jj & 1)), (jj >> 1) & 1, prm.wait_cycles);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- CUDA-core work
        const uint32_t MASK = 0xffffffffu;
        const int wq = warp & 3;                   // TMEM lane quarter = 32-row quarter of the block
        const int g = warp >> 2;                   // column group: TMEM columns [32 g, 32 g + 32) of G, S, Y
        const int hs = g >> 1, ch = g & 1;         // head of the column group, its half of headdim
        const int r = wq * 32 + lane;              // row in block == TMEM lane (token row, or state index n)
        const int h = h0 + hs;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);

        // cX of block jj (rows scaled in place by c, this group's 4 chunks of its row) and the
        // starting value D x / r of its Y accumulator
        auto cx_pass = [&](int jj) -> bool {
            const int st = jj & 1, sl = jj % 3;
            if (!mbar_wait(bar(B_TABREADY0 + sl), (jj / 3) & 1, MASK, abort_flag, prm.status, 41)) return false;
            if (!mbar_wait(bar(B_XFULL0 + st), (jj >> 1) & 1, MASK, abort_flag, prm.status, 42)) return false;
            // Y buffer st was last read by block jj-2's epilogue, which this warp ran before this
            // pass, on the same TMEM lanes and columns it writes here (each warp its own slice)
            const float *tb = tab_s + sl * kTabFloats;
            const float cf = tb[kTabCF + hs * kBlk + r], dr = tb[kTabDR + hs * kBlk + r];
            uint8_t *xt = sm + kOffX + st * kPairBytes + hs * kTileBytes;
            float dx[32];
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int q = 4 * ch + qq;
                const uint4 v = *reinterpret_cast<const uint4 *>(xt + swz(r, q));
                const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float lo = bf16lo(xw[i]), hi = bf16hi(xw[i]);
                    o[i] = pack_bf16(lo * cf, hi * cf);
                    dx[8 * qq + 2 * i] = lo * dr;
                    dx[8 * qq + 2 * i + 1] = hi * dr;
                }
                *reinterpret_cast<uint4 *>(xt + swz(r, q)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            tmem_st32f_nw(tl + kColY + 128u * st + 32 * g, dx);
            fence_async_smem();                // cX is read by the tensor core
            tmem_wait_st();
            tc_fence_before();                 // Y's starting value is read by the MMA
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_CXREADY0 + st));
            return true;
        };

        // Gc of block j: G masked to the causal triangle (memory order: sources s <= r forward,
        // s >= r reverse), bf16, written in place: K-step ks (16 sources) at columns [16 ks, 16 ks + 8)
        auto mask_pass = [&]() {
            const bool all = dir > 0 ? g < wq : g > wq;     // source quarter g wholly inside the triangle
            const bool diag = g == wq;
            uint32_t m[16];
            if (all || diag) {
                float gv[32];
                tmem_ld32(tl + kColG + 32 * g, gv);
#pragma unroll
                for (int i = 0; i < 16; ++i) m[i] = pack_bf16(gv[2 * i], gv[2 * i + 1]);
                if (diag) {
                    // keep sources u <= lane (forward) or u >= lane (reverse): bit u of keep.
                    // Applied to the packed words with integer masks, without branches.
                    const uint32_t low = lane == 31 ? 0xffffffffu : (2u << lane) - 1u;
                    const uint32_t keep = dir > 0 ? low : ~((1u << lane) - 1u);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t k2 = keep >> (2 * i);
                        m[i] &= ((k2 & 1u) * 0xffffu) | (((k2 >> 1) & 1u) * 0xffff0000u);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) m[i] = 0u;
            }
            tmem_st8_nw(tl + kColG + 32 * g, m);
            tmem_st8_nw(tl + kColG + 32 * g + 16, m + 8);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_GCREADY));
        };

        // state hand-off into block jn: S (state after block jn-1, divided by its kappa) is scaled
        // by e^{m_jn} kappa_{jn-1} in place, and its bf16 copy (rows = n) is the B operand of the
        // next Y_off.  k2p = kappa exponent of block jn-1.
        auto state_pass = [&](int jn, float k2p) -> bool {
            if (!mbar_wait(bar(B_TABREADY0 + jn % 3), (jn / 3) & 1, MASK, abort_flag, prm.status, 48)) return false;
            // the bf16 copy is read by Y_off of block jn-1 (stream B commits B_YOFFDONE every block)
            if (!mbar_wait(bar(B_YOFFDONE), (jn - 1) & 1, MASK, abort_flag, prm.status, 50)) return false;
            const float m2n = tab_s[(jn % 3) * kTabFloats + kTabM2 + hs];
            const float l2 = m2n + k2p;
            float sv[32];
            tmem_ld32(tl + kColS + 32 * g, sv);
            if (l2 >= -120.f) {
                const float f = ex2_ftz(l2);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] *= f;
            } else {
                // the product of the two factors would leave float range: apply them one by one
                const float f1 = ex2_ftz(m2n), f2 = ex2_ftz(k2p);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = (sv[i] * f1) * f2;
            }
            tmem_st32f_nw(tl + kColS + 32 * g, sv);
            uint8_t *stile = sm + kOffS + hs * kTileBytes;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint4 o;
                o.x = pack_bf16(sv[8 * qq + 0], sv[8 * qq + 1]);
                o.y = pack_bf16(sv[8 * qq + 2], sv[8 * qq + 3]);
                o.z = pack_bf16(sv[8 * qq + 4], sv[8 * qq + 5]);
                o.w = pack_bf16(sv[8 * qq + 6], sv[8 * qq + 7]);
                *reinterpret_cast<uint4 *>(stile + swz(r, 4 * ch + qq)) = o;
            }
            fence_async_smem();                // the copy is read by the tensor core
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SREADY));
            return true;
        };

        // state entering or leaving the scan, [b][h][p][n] float32: this thread's row is n = r, its
        // columns p = 32 ch + i (consecutive lanes read consecutive n: coalesced)
        const size_t sslot = ((size_t)b * prm.H + h) * kP * kN;
        // state entering the scan: scaled by e^{m_0} into TMEM, with its bf16 copy for block 0's Y_off
        auto init_pass = [&]() {
            float sv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = prm.s_in ? prm.s_in[sslot + (size_t)(32 * ch + i) * kN + r] : 0.f;
            // S_in <- exp(A T_piece) S_in + S_loc(piece), over the pieces of the segments before
            // this one, in scan order
            const size_t chain = ((size_t)b * prm.H + h) * 2 + slot;
            const int npieces = (prm.nseg - 1) * prm.npiece;
            for (int s2 = 0; s2 < seg * prm.npiece; ++s2) {
                const float d2 = ex2_ftz(prm.ldec[chain * npieces + s2]);
                const float *sl = prm.sloc + (chain * npieces + s2) * kP * kN;
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = sv[i] * d2 + sl[(size_t)(32 * ch + i) * kN + r];
            }
            const float f = ex2_ftz(tab_s[kTabM2 + hs]);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] *= f;
            tmem_st32f_nw(tl + kColS + 32 * g, sv);
            uint8_t *stile = sm + kOffS + hs * kTileBytes;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint4 o;
                o.x = pack_bf16(sv[8 * qq + 0], sv[8 * qq + 1]);
                o.y = pack_bf16(sv[8 * qq + 2], sv[8 * qq + 3]);
                o.z = pack_bf16(sv[8 * qq + 4], sv[8 * qq + 5]);
                o.w = pack_bf16(sv[8 * qq + 6], sv[8 * qq + 7]);
                *reinterpret_cast<uint4 *>(stile + swz(r, 4 * ch + qq)) = o;
            }
            fence_async_smem();
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SREADY));
        };

        // prologue: cX of block 0, the entering state
        bool ok = nblk == 0 || cx_pass(0);
        if (ok && has_in && nblk > 0) init_pass();
        for (int j = 0; j < nblk && ok; ++j) {
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            SSD_TRACE_PT(warp, j, 0);
            const int st = j & 1, sl = j % 3;
            // (1) mask this block's scores
            if (!mbar_wait(bar(B_GFULL), j & 1, MASK, abort_flag, prm.status, 44)) break;
            SSD_TRACE_PT(warp, j, 1);
            tc_fence_after();
            mask_pass();
            SSD_TRACE_PT(warp, j, 2);
            SSD_TRACE_PT(warp, j, 3);
            if (j + 1 < nblk) {
                // (2) the state hand-off into the next block
                const float k2 = tab_s[sl * kTabFloats + kTabK2 + hs];
                if (!mbar_wait(bar(B_STFULL), j & 1, MASK, abort_flag, prm.status, 45)) break;
                SSD_TRACE_PT(warp, j, 4);
                tc_fence_after();
                if (!state_pass(j + 1, k2)) break;
                SSD_TRACE_PT(warp, j, 5);
            } else if (s_out) {
                // state leaving the scan: S_out = kappa_last * S (after the last state product)
                if (!mbar_wait(bar(B_STFULL), j & 1, MASK, abort_flag, prm.status, 49)) break;
                tc_fence_after();
                const float f = ex2_ftz(tab_s[sl * kTabFloats + kTabK2 + hs]);
                float sv[32];
                tmem_ld32(tl + kColS + 32 * g, sv);
#pragma unroll
                for (int i = 0; i < 32; ++i) s_out[sslot + (size_t)(32 * ch + i) * kN + r] = sv[i] * f;
            }
            // (3) epilogue: y = r Y_j in bf16 into this block's B buffer, which G and the state
            // product have consumed (the state product's completion was awaited in (2), or here
            // for the last block); the store warp writes the tiles to y.  It comes before the next
            // block's cX pass: the sooner the tiles leave, the sooner B of block j+2 can be loaded
            // into this buffer, and the next G waits for that B.
            if (j + 1 == nblk && !s_out && !mbar_wait(bar(B_STFULL), j & 1, MASK, abort_flag, prm.status, 49))
                break;
            if (!mbar_wait(bar(B_YFULL), j & 1, MASK, abort_flag, prm.status, 46)) break;
            SSD_TRACE_PT(warp, j, 7);
            tc_fence_after();
            {
                const float rr = tab_s[sl * kTabFloats + kTabR + hs * kBlk + r];
                float yv[32];
                tmem_ld32(tl + kColY + 128u * st + 32 * g, yv);
                uint8_t *yt = sm + kOffB + st * kPairBytes + hs * kTileBytes;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint4 ov;
                    ov.x = pack_bf16(rr * yv[8 * qq + 0], rr * yv[8 * qq + 1]);
                    ov.y = pack_bf16(rr * yv[8 * qq + 2], rr * yv[8 * qq + 3]);
                    ov.z = pack_bf16(rr * yv[8 * qq + 4], rr * yv[8 * qq + 5]);
                    ov.w = pack_bf16(rr * yv[8 * qq + 6], rr * yv[8 * qq + 7]);
                    *reinterpret_cast<uint4 *>(yt + swz(r, 4 * ch + qq)) = ov;
                }
            }
            fence_async_smem();                // the tile is read by a TMA store
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_TABFREE0 + sl));     // and the block's tables, for the last time
                mbar_arrive(bar(B_TILE0 + st));
            }
            SSD_TRACE_PT(warp, j, 8);
            if (j + 1 < nblk) {
                // (4) the next block's cX and Y starting value (its x stage was loaded once block
                // j-1's products had read the stage: placed here, the load has most of a block)
                if (!cx_pass(j + 1)) break;
                SSD_TRACE_PT(warp, j, 6);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    SSD_TRACE_CTA(1);
    if (warp == kWarpMmaA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

}  // namespace

size_t tcs_smem_bytes() { return kSmemBytes; }

#ifdef SSD_TRACE
extern "C" int ssd_debug_cta_times(unsigned long long *out, int n) {
    if (n < 4096 * 3) return -1;
    return cudaMemcpyFromSymbol(out, g_cta_time, sizeof(unsigned long long) * 4096 * 3) == cudaSuccess ? 4096 : -2;
}
extern "C" int ssd_debug_blocks(unsigned long long *out, int n) {
    const int total = 2 * kTraceAllBlocks * 4;
    if (n < total) return -1;
    return cudaMemcpyFromSymbol(out, g_blk, sizeof(unsigned long long) * total) == cudaSuccess ? total : -2;
}
extern "C" int ssd_debug_trace(unsigned long long *out, int n) {
    const int total = kTraceWarps * kTraceBlocks * kTracePts;
    if (n < total) return -1;
    return cudaMemcpyFromSymbol(out, g_trace, sizeof(unsigned long long) * total) == cudaSuccess ? total : -2;
}
#endif

// Launches the shared-score kernel for the chains it can run (the steep ones are the exact
// kernel's).
cudaError_t launch_tcs(const TcArgs &t, bool bidir, void *y, unsigned long long *ticket, unsigned long long *ready,
                       const SegScratch &sc, unsigned long long epoch, cudaStream_t st) {
    // The shared-memory opt-in belongs to the kernel in the current context: set on every launch
    // (a host-side call), so it holds in any context the caller makes current.
    cudaError_t e = cudaFuncSetAttribute(k_ssd_tcs, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int ndir = bidir ? 2 : 1;
    const uint64_t rows = (uint64_t)t.batch * t.L;
    TcsMaps maps;
    memset(&maps, 0, sizeof maps);
    TcsParams p{};
    for (int s = 0; s < ndir; ++s) {
        const TcDir &d = t.d[s];
        if (!make_map(&maps.x[s], d.x, rows, (uint64_t)t.H * kP, 64, true) ||
            !make_map(&maps.dt[s], d.dt, rows, (uint64_t)t.H, 8, false) ||
            !make_map(&maps.b[s], d.B, rows, kN, 64, true) || !make_map(&maps.c[s], d.C, rows, kN, 64, true))
            return cudaErrorInvalidValue;
        p.d[s].A = d.A;
        p.d[s].D = d.D;
        p.d[s].dt = static_cast<const __nv_bfloat16 *>(d.dt);
    }
    if (!make_map(&maps.y, y, rows, (uint64_t)t.H * kP, 64, true)) return cudaErrorInvalidValue;
    p.batch = t.batch; p.L = t.L; p.H = t.H; p.nblk = t.L / kBlk;
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.bidir = bidir ? 1 : 0;
    p.dir_single = t.d[0].dir;
    p.status = t.status;
    p.ticket = ticket;
    p.ready = ready;
    p.epoch = epoch;
    p.wait_cycles = t.wait_cycles;
    p.fault = t.fault;
    p.s_in = bidir ? nullptr : t.s_in;
    p.s_out = bidir ? nullptr : t.s_out;
    p.nseg = t.nseg > 1 ? t.nseg : 1;
    p.sb = tc_segment_blocks(t.L, p.nseg);
    p.npiece = t.npiece;
    p.sloc = sc.sloc;
    p.ldec = sc.ldec;
    p.steep = sc.steep;
    const int grid = t.batch * (t.H / 2) * p.nseg * ndir;
    k_ssd_tcs<<<grid, kThreads, kSmemBytes, st>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace ssd
