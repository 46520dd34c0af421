// ssd_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) path of the SSD scan for
// bf16 io, headdim 64, d_state 128, one B/C group shared by a head pair.
//
// One CTA owns (batch b, head pair {h0, h0+1}, direction) and walks the
// sequence in scan order in blocks of 128 tokens, carrying the float32 state
// of both heads in TMEM.  Per block (rows r = 0..127 in memory order, TMEM
// lane r = token t0 + r), with cs the cumulative A*dt in scan order:
//
//   tables: cs, dt, decay factors      CUDA cores, from a dt ring loaded one block ahead;
//                                      written during the previous block's Y_diag MMA
//                                      (smem, 2 buffers)
//   G      = C B^T                     tcgen05, shared by both heads   TMEM [0,128)
//   M_h    = G (.) decay_h (.) dt      CUDA cores, bf16, written over the G columns it
//                                      came from (A operand of the intra-block MMA)
//   Y_off  = C S'^T                    tcgen05, N = 2 heads x 64       TMEM [384,512)
//                                      (S' = state entering the block, bf16 copy in smem)
//   S'    <- exp(cs_last) S'           CUDA cores, in place in TMEM [128,256)
//   S'    += B^T (w (.) X)             tcgen05, N = 2 heads x 64, accumulates into S'
//   Y_diag = D x + M_h X_h             D x stored by the CUDA cores in the w (.) x pass,
//                                      then tcgen05, A from TMEM, N = 64    TMEM [256,384)
//   y      = Y_diag + exp(cs_r) Y_off  CUDA cores -> smem tile -> TMA store
//
// This is the chunked evaluation of the recurrence S <- exp(dt A) S +
// dt x (outer) B, y = C.S + D x that the Mamba-2 layers of the DiffuMamba
// mixer ("DiffuMamba", technical summary, section 2) and the R2LM
// right-to-left stream ("Bifocal Diffusion Language Models", section 2,
// mechanism) run.  The reverse direction walks the blocks from the end and
// uses suffix sums and the upper triangle: the flip lives in the address
// arithmetic only.
//
// Decay mask.  Inside a block the 128 rows split into four 32-row quarters
// (= the four TMEM lane quarters).  For a source s in an earlier quarter than
// the output row r, exp(cs_r - cs_s) = exp(cs_r - cs_ref) * exp(cs_ref - cs_s)
// with ref the quarter boundary between them; both factors are <= 1, so the
// product never overflows, and the mask becomes (row factor) x (column table)
// with no exponential per element.  Inside the diagonal quarter the same is done
// at 16-row granularity: exp(cs_r - cs_s) = R16[r] * D16[s] within one 16-row
// sub-block (masked to the causal half) and R16[r] * O16[s] from the sub-block
// before.  D16 grows across its sub-block, so a sub-block whose decay exceeds
// 2^120 falls back to one exponential per element.
//
// Bidirectional mixer in one launch.  The CTAs of the forward and reverse
// scans of one head pair are neighbours in the grid.  For every output block
// the first of the two to finish writes its part of y, the second adds its
// own part to it: an epoch-tagged ticket per (batch, head, block), taken by a
// store warp once the block's part is complete, decides the order, and an
// epoch-tagged ready word publishes the first part.  The first never waits,
// and a second only waits for a first that has already passed every earlier
// block of its own walk, so the hand-off cannot deadlock whatever the residency.
//
// Warp roles (640 threads): warps 0-15 form four warpgroups doing the CUDA-core
// work (thread r <-> TMEM lane r; warpgroup g = 2*head + column half), warp 16
// issues the TMA loads, warp 17 owns TMEM and issues the MMAs (one thread),
// warps 18 and 19 write y for heads h0 and h0+1 (TMA stores, and the
// forward/reverse hand-off), so the CUDA-core warps never wait on global memory.  Every wait is
// bounded; a wait that runs out records SSD_ERR_TIMEOUT in the status word and
// the CTA winds down without touching more data.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <chrono>
#include <cstring>
#include <mutex>

#include "ssd_tc.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kBlk = 128;            // tokens per block (MMA M)
constexpr int kP = 64, kN = 128;
constexpr int kThreads = 640;        // warps 0-15: four warpgroups; 16: TMA; 17: MMA + TMEM;
                                     // 18-19: decay tables and y stores, one warp per head
constexpr int kWarpTma = 16, kWarpMma = 17, kWarpStore = 18;
constexpr uint32_t kTileBytes = kBlk * 64 * 2;        // one [128][64] bf16 swizzled tile = 16 KB
constexpr uint32_t kDtBytes = kBlk * 8 * 2;           // dt box: 128 tokens x 8 heads, bf16
constexpr uint32_t kStageBytes = 2 * kTileBytes;      // x of 2 heads = 32 KB

// TMEM column map: G (then M over it), running state S', Y_diag, Y_off
constexpr uint32_t kColG = 0, kColST = 128, kColYD = 256, kColYO = 384;

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffX = 0;                          // 2 stages: [x h0 | x h1]
constexpr uint32_t kOffB = kOffX + 2 * kStageBytes;    // 2 sub-tiles (n 0..63, 64..127)
constexpr uint32_t kOffC = kOffB + 2 * kTileBytes;
constexpr uint32_t kOffWX = kOffC + 2 * kTileBytes;    // 2 heads
constexpr uint32_t kOffSP = kOffWX + 2 * kTileBytes;   // 2 heads, rows = state index n
// Decay tables of one block, both heads (float, log2 units where noted), double-buffered by
// block parity: the CUDA-core warps write block j+1's while the tensor core computes block
// j's intra-block output.
constexpr uint32_t kTabCS = 0;                          // cs2[2][128]: cs_r * log2 e, scan order
constexpr uint32_t kTabDT = kTabCS + 2 * kBlk;          // dt[2][128]
constexpr uint32_t kTabW = kTabDT + 2 * kBlk;           // W[2][4][128]: off-diagonal column factors
constexpr uint32_t kTabE1 = kTabW + 8 * kBlk;           // e1[2][128]: off-diagonal row factors
constexpr uint32_t kTabWR = kTabE1 + 2 * kBlk;          // wr[2][128]: weight of row r in the block state
constexpr uint32_t kTabER = kTabWR + 2 * kBlk;          // er[2][128]: decay from the block start to row r
constexpr uint32_t kTabR16 = kTabER + 2 * kBlk;        // R16[2][128]: row factor to the 16-row sub-block start
constexpr uint32_t kTabD16 = kTabR16 + 2 * kBlk;       // D16[2][128]: column factor, same sub-block
constexpr uint32_t kTabO16 = kTabD16 + 2 * kBlk;       // O16[2][128]: column factor, next sub-block
constexpr uint32_t kTabBig = kTabO16 + 2 * kBlk;       // big[2][8]: sub-block needs exact exponentials
constexpr uint32_t kTabA = kTabBig + 16;               // ablk[2]: decay across the block
constexpr uint32_t kTabFloats = kTabA + 4;
constexpr uint32_t kOffTab = kOffSP + 2 * kTileBytes;   // 2 buffers
constexpr uint32_t kOffDT = (kOffTab + 2 * kTabFloats * 4 + 127) / 128 * 128;   // dt ring, 2 slots
constexpr uint32_t kOffBar = kOffDT + 2 * kDtBytes;
constexpr uint32_t kNumBars = 25;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag, wait limit, steep flag
constexpr uint32_t kSmemBytes = kOffMisc + 32 + 1024;  // + alignment slack
static_assert(kStageBytes % 1024 == 0, "x tiles must stay 1024-byte aligned");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Every barrier completes at most once more before each of its waiters has
// passed its wait for the previous completion (a waiter tells completions
// apart by phase parity only).  Where a producer could otherwise run two
// completions ahead, the barrier is per buffer: B_TILE (per head and x stage),
// B_TABREADY (per table buffer), B_DTFULL and B_DTEMPTY (per dt slot).
enum Bar {
    B_XFULL0 = 0, B_XFULL1, B_XEMPTY0, B_XEMPTY1, B_BCFULL, B_BCEMPTY, B_GFULL, B_WXREADY, B_SPREADY, B_STFULL,
    B_MREADY, B_YFULL, B_YEMPTY, B_DONE, B_TILE00, B_TILE01, B_TILE10, B_TILE11, B_TABREADY0, B_TABREADY1,
    B_DTFULL0, B_DTFULL1, B_DTEMPTY0, B_DTEMPTY1, B_YFULLH0
};

constexpr float kLog2e = 1.4426950408889634f;


struct TcDirParams {
    const float *A, *D;
    const __nv_bfloat16 *dt;
};

struct TcParams {
    const unsigned long long *steep;    // [batch][H/2][2], epoch-tagged: the chains this kernel runs
    int batch, L, H, nblk;
    int bidir;                          // 1: slot = blockIdx & 1, forward/reverse hand-off through flags
    int dir_single;                     // direction of slot 0 when bidir == 0
    TcDirParams d[2];
    __nv_bfloat16 *y;
    int *status;
    unsigned long long *ticket;         // [batch][H][nblk], epoch-tagged
    unsigned long long *ready;          // [batch][H][nblk], epoch-tagged
    unsigned long long epoch;
    long long wait_cycles;              // bound of every device-side wait
    int fault;                          // test hook: 1 = the first direction never publishes its part
    const float *s_in;                  // single direction: [batch][H][P][N] state entering the scan, or null
    float *s_out;                       // single direction: [batch][H][P][N] state leaving the scan, or null
};

struct TcMaps {
    CUtensorMap x[2], dt[2], b[2], c[2], y;
};

// ------------------------------------------------------------------ the kernel

// kState: the state may enter and leave the call (single-direction scan with a carried state);
// the instantiation without it is the one the bidirectional mixer and plain scans run.
template <bool kState>
__global__ void __launch_bounds__(kThreads, 1) k_ssd_tc(const __grid_constant__ TcMaps maps, const __grid_constant__ TcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    float *tab_s = reinterpret_cast<float *>(sm + kOffTab);         // [2 buffers][kTabFloats]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npairs = prm.H / 2;
    const int unit = prm.bidir ? (blockIdx.x >> 1) : blockIdx.x;
    const int slot = prm.bidir ? (blockIdx.x & 1) : 0;
    const int dir = prm.bidir ? (slot == 0 ? 1 : -1) : prm.dir_single;
    const int b = unit / npairs, hp = unit % npairs;
    const int h0 = 2 * hp;
    const int nblk = prm.nblk, L = prm.L;
    const int has_in = kState && prm.s_in != nullptr;   // a state enters the scan (single direction)
    const CUtensorMap *map_x = &maps.x[slot], *map_dt = &maps.dt[slot], *map_b = &maps.b[slot],
                      *map_c = &maps.c[slot];

    // The CTA past the last chain: wait for the shared-score grid this launch may overlap, so
    // that this grid completes after it (a no-op when launched in plain stream order).
    if ((int)blockIdx.x == (prm.bidir ? 2 : 1) * prm.batch * npairs) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        return;
    }
    // This kernel runs only the chains the shared-score kernel leaves: those the steep-decay
    // marks of this call name (one pass, before both kernels, decides for every chain)
    if (*reinterpret_cast<const volatile unsigned long long *>(prm.steep + ((size_t)b * npairs + h0 / 2) * 2 + slot) !=
        prm.epoch)
        return;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        // arrival counts: 16 = one per CUDA-core warp, 8 = one per warp of a head's two
        // warpgroups, 1 = one thread (the store warp's, for the x stages) / one MMA commit
        constexpr uint32_t k16 = (1u << B_WXREADY) | (1u << B_SPREADY) | (1u << B_MREADY) | (1u << B_YEMPTY) |
                                 (1u << B_TABREADY0) | (1u << B_TABREADY1) | (1u << B_DTEMPTY0) | (1u << B_DTEMPTY1);
        constexpr uint32_t k8 = (1u << B_TILE00) | (1u << B_TILE01) | (1u << B_TILE10) | (1u << B_TILE11);
        for (int i = 0; i < (int)kNumBars; ++i) mbar_init(bar(i), (k16 >> i) & 1 ? 16 : (k8 >> i) & 1 ? 8 : 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint32_t MASK = 1u;
            int issued = 0;   // blocks whose loads were issued
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_x)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_dt)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_b)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map_c)) : "memory");
            // dt of block jj into slot jj & 1 of the dt ring (one block ahead of x)
            int dt_issued = 0, x_issued = 0;
            auto load_dt = [&](int jj) -> bool {
                const int sl = jj & 1;
                if (jj >= 2 && !mbar_wait(bar(B_DTEMPTY0 + sl), ((jj >> 1) - 1) & 1, MASK, abort_flag, prm.status, 13))
                    return false;
                const int cmj = dir > 0 ? jj : nblk - 1 - jj;
                mbar_expect_tx(bar(B_DTFULL0 + sl), kDtBytes);
                tma_load_2d(sbase + kOffDT + sl * kDtBytes, map_dt, h0 & ~7, b * L + cmj * kBlk, bar(B_DTFULL0 + sl));
                dt_issued = jj + 1;
                return true;
            };
            bool ok = load_dt(0);
            for (int j = 0; j < nblk && ok; ++j) {
                const int cm = dir > 0 ? j : nblk - 1 - j;
                const int row = b * L + cm * kBlk;
                const int st = j & 1;
                if (j >= 2 && !mbar_wait(bar(B_XEMPTY0 + st), ((j >> 1) - 1) & 1, MASK, abort_flag, prm.status, 11)) break;
                const uint32_t stage = sbase + kOffX + st * kStageBytes;
                mbar_expect_tx(bar(B_XFULL0 + st), kStageBytes);
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(stage + h * kTileBytes, map_x, (h0 + h) * kP, row, bar(B_XFULL0 + st));
                x_issued = j + 1;
                if (j + 1 < nblk && !load_dt(j + 1)) break;
                if (j >= 1 && !mbar_wait(bar(B_BCEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 12)) break;
                mbar_expect_tx(bar(B_BCFULL), 4 * kTileBytes);
                for (int q = 0; q < 2; ++q) {
                    tma_load_2d(sbase + kOffB + q * kTileBytes, map_b, q * 64, row, bar(B_BCFULL));
                    tma_load_2d(sbase + kOffC + q * kTileBytes, map_c, q * 64, row, bar(B_BCFULL));
                }
                issued = j + 1;
            }
            if (*abort_flag) {
                // let copies still in flight land before the CTA exits: the last two x stages,
                // the last B/C load and the last two dt slots
                for (int jj = x_issued - 1; jj >= 0 && jj >= x_issued - 2; --jj)
                    mbar_drain(bar(B_XFULL0 + (jj & 1)), (jj >> 1) & 1, prm.wait_cycles);
                if (issued > 0) mbar_drain(bar(B_BCFULL), (issued - 1) & 1, prm.wait_cycles);
                for (int jj = dt_issued - 1; jj >= 0 && jj >= dt_issued - 2; --jj)
                    mbar_drain(bar(B_DTFULL0 + (jj & 1)), (jj >> 1) & 1, prm.wait_cycles);
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t MASK = 1u;
            const uint32_t id_g = idesc(128, 0, 0), id_s = idesc(128, 1, 1), id_yo = idesc(128, 0, 1),
                           id_yd = idesc(64, 0, 1);
            const uint32_t aB = sbase + kOffB, aC = sbase + kOffC, aWX = sbase + kOffWX, aSP = sbase + kOffSP;
            for (int j = 0; j < nblk; ++j) {
                const int st = j & 1;
                const uint32_t aX = sbase + kOffX + st * kStageBytes;
                // G = C B^T  (M = rows, N = source rows, K = n)
                if (!mbar_wait(bar(B_BCFULL), j & 1, MASK, abort_flag, prm.status, 21)) break;
                // the previous block's M (read by its intra-block MMA) occupies the G columns
                if (j >= 1 && !mbar_wait(bar(B_YFULL), (j - 1) & 1, MASK, abort_flag, prm.status, 22)) break;
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                    mma_ss(tmem + kColG, sdesc(aC + off, 16, 1024), sdesc(aB + off, 16, 1024), id_g, ks > 0);
                }
                mma_commit(bar(B_GFULL));
                if (j >= 1 || has_in) {
                    // Y_off = C S'^T of the state entering this block (M = rows, N = (head, p), K = n);
                    // SP holds bf16(S') and the float32 state has been scaled by this block's decay
                    if (!mbar_wait(bar(B_SPREADY), (j - 1 + has_in) & 1, MASK, abort_flag, prm.status, 23)) break;
                    // the previous block's epilogue has read both Y accumulators
                    if (j >= 1 && !mbar_wait(bar(B_YEMPTY), (j - 1) & 1, MASK, abort_flag, prm.status, 24)) break;
                    tc_fence_after();
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t offc = (ks >> 2) * kTileBytes + (ks & 3) * 32;
                        mma_ss(tmem + kColYO, sdesc(aC + offc, 16, 1024), sdesc(aSP + ks * 2048, kTileBytes, 1024),
                               id_yo, ks > 0);
                    }
                }
                // S'^T (+)= B^T (w x)  (M = n, N = (head, p), K = rows); both operands MN-major
                if (!mbar_wait(bar(B_WXREADY), j & 1, MASK, abort_flag, prm.status, 25)) break;
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = ks * 2048;
                    mma_ss(tmem + kColST, sdesc(aB + off, kTileBytes, 1024), sdesc(aWX + off, kTileBytes, 1024), id_s,
                           (j > 0) || has_in || (ks > 0));
                }
                mma_commit(bar(B_STFULL));
                mma_commit(bar(B_BCEMPTY));
                // Y_diag += M_h X_h  (A from TMEM, B = X_h MN-major, N = 64 per head), on top of
                // the D x the CUDA-core warps stored there in their w.x pass
                if (!mbar_wait(bar(B_MREADY), j & 1, MASK, abort_flag, prm.status, 27)) break;
                if (!mbar_wait(bar(B_XFULL0 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 29)) break;
                tc_fence_after();
                for (int h = 0; h < 2; ++h) {
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ts(tmem + kColYD + 64 * h, tmem + kColG + 16 * ks + 8 * h,
                               sdesc(aX + h * kTileBytes + ks * 2048, kTileBytes, 1024), id_yd, 1);
                    // head 0's warps can start their epilogue while head 1's MMAs run
                    if (h == 0) mma_commit(bar(B_YFULLH0));
                }
                mma_commit(bar(B_YFULL));
            }
            // drain: every MMA issued above has completed before TMEM is released
            mma_commit(bar(B_DONE));
            mbar_drain(bar(B_DONE), 0, prm.wait_cycles);
        }
    } else if (warp == kWarpStore) {
        // ---------------------------------------------------------- y stores of both heads
        // The two directions of a head pair take one ticket per output block, at the pair's
        // first head: the same word the shared-score kernel takes, so a pair whose two chains
        // run in different kernels (one direction steep, the other not) still meets once per
        // block.  The first direction stores both heads' tiles and publishes the pair once both
        // have landed; the second waits for that and adds both.  (Warp kWarpStore + 1 has no
        // part in this.)
        const uint32_t MASK = 0xffffffffu;
        const size_t pair_base = ((size_t)b * prm.H + h0) * nblk;
        for (int j = 0; j < nblk; ++j) {
            const int st = j & 1;
            const int cm = dir > 0 ? j : nblk - 1 - j;
            if (!mbar_wait(bar(B_TILE00 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 61)) break;
            if (!mbar_wait(bar(B_TILE10 + st), (j >> 1) & 1, MASK, abort_flag, prm.status, 62)) break;
            const uint32_t tile = sbase + kOffX + st * kStageBytes;
            int sec = 0;
            if (prm.bidir) {
                if (lane == 0) {
                    // this direction's part of the block is complete: first or second?
                    sec = atomicExch(prm.ticket + pair_base + cm, prm.epoch) == prm.epoch;
                    if (sec) {
                        // the other direction took the block first and is storing it
                        const unsigned long long *rp = prm.ready + pair_base + cm;
                        const long long t0 = clock64();
                        while (ld_acquire(rp) != prm.epoch) {
                            if (*abort_flag) { sec = 2; break; }
                            if (clock64() - t0 > prm.wait_cycles) {
                                *abort_flag = 1;
                                atomicExch(prm.status, 47);
                                sec = 2;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                }
                sec = __shfl_sync(MASK, sec, 0);
                if (sec == 2) break;
            }
            if (lane == 0) {
                if (sec == 0) {
                    for (int hs = 0; hs < 2; ++hs)
                        tma_store_2d(&maps.y, tile + hs * kTileBytes, (h0 + hs) * kP, b * L + cm * kBlk);
                } else {
                    // y += this part: bulk tensor reductions (bf16 add in L2) onto the published part
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    for (int hs = 0; hs < 2; ++hs)
                        tma_reduce_add_2d(&maps.y, tile + hs * kTileBytes, (h0 + hs) * kP, b * L + cm * kBlk);
                }
                bulk_commit();
                bulk_wait_read0();                        // the tiles may be overwritten from here on
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_XEMPTY0 + st));
                if (prm.bidir && sec == 0) {
                    bulk_wait0();                         // both heads' parts are in global memory
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    if (prm.fault != 1) st_release(prm.ready + pair_base + cm, prm.epoch);
                }
            }
        }
        if (lane == 0) bulk_wait0();                      // every store has landed before the CTA exits
    } else if (warp == kWarpStore + 1) {
        // no work: the store warp above writes both heads
    } else {
        // ---------------------------------------------------------- CUDA-core work
        // Four warpgroups: g = 2 * head + half.  Each handles one head's rows and one half
        // (32 of 64) of its headdim columns in the per-head passes, and a quarter of the
        // 16-source K-steps (both heads) in the decay-mask pass.
        const uint32_t MASK = 0xffffffffu;
        const int g = warp >> 2;                   // warpgroup 0..3
        const int hs = g >> 1, c = g & 1;          // head within the pair, column half
        const int wq = warp & 3;                   // TMEM lane quarter = 32-row quarter of the block
        const int r = wq * 32 + lane;              // row in block == TMEM lane
        const int h = h0 + hs;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        const float Dh = prm.d[slot].D ? prm.d[slot].D[h] : 0.f;
        uint8_t *wx_tile = sm + kOffWX + hs * kTileBytes;
        uint8_t *sp_tile = sm + kOffSP + hs * kTileBytes;
        const uint32_t colST = kColST + 64 * hs + 32 * c, colYD = kColYD + 64 * hs + 32 * c,
                       colYO = kColYO + 64 * hs + 32 * c;

        // Decay tables of block jj (into buffer jj & 1) from the dt ring.  Thread (r, head hs)
        // computes the cumulative A dt of its row in scan order (prefix over rows forward, suffix
        // reverse; log2 units) and writes its share of the row's entries: half c = 0 the mask
        // tables, half c = 1 the w.x, epilogue and sub-block factors.
        const float A2 = prm.d[slot].A[h] * kLog2e;   // log2 units: exp(a) = exp2(a * log2 e)
        auto make_tables = [&](int jj) -> bool {
            const int sl = jj & 1;
            if (!mbar_wait(bar(B_DTFULL0 + sl), (jj >> 1) & 1, MASK, abort_flag, prm.status, 51)) return false;
            // buffer jj & 1 was last read in block jj - 2: every warp has finished its epilogue
            if (jj >= 2 && !mbar_wait(bar(B_YEMPTY), (jj - 2) & 1, MASK, abort_flag, prm.status, 52)) return false;
            const __nv_bfloat16 *dtt = reinterpret_cast<const __nv_bfloat16 *>(sm + kOffDT + sl * kDtBytes);
            const float d = __bfloat162float(dtt[r * 8 + (h & 7)]);
            float s = d;                                   // inclusive scan inside the quarter
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = dir > 0 ? __shfl_up_sync(MASK, s, o) : __shfl_down_sync(MASK, s, o);
                if (dir > 0 ? lane >= o : lane + o < 32) s += u;
            }
            float tot[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float v = __bfloat162float(dtt[(32 * q + lane) * 8 + (h & 7)]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(MASK, v, o);
                tot[q] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_DTEMPTY0 + sl));      // dt slot read: free for block jj + 2
            // base[q] = sum of the quarters before q in scan order (cs just before quarter q)
            float base[4], acc = 0.f;
            if (dir > 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) { base[q] = acc; acc += tot[q]; }
            } else {
#pragma unroll
                for (int q = 3; q >= 0; --q) { base[q] = acc; acc += tot[q]; }
            }
            const float own_base = wq == 0 ? base[0] : wq == 1 ? base[1] : wq == 2 ? base[2] : base[3];
            const float own_tot = wq == 0 ? tot[0] : wq == 1 ? tot[1] : wq == 2 ? tot[2] : tot[3];
            const float c2 = A2 * (own_base + s);
            const float cl2 = A2 * acc;                    // cs at the block's last scan position
            float *tb = tab_s + sl * kTabFloats;
            if (c == 0) {
                tb[kTabCS + hs * kBlk + r] = c2;
                tb[kTabDT + hs * kBlk + r] = d;
                // column factors for the later quarters: W[q2][s] = exp(cs_ref(q2) - cs_s) dt_s
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const bool off = dir > 0 ? wq < q2 : wq > q2;
                    if (off) tb[kTabW + (hs * 4 + q2) * kBlk + r] = ex2_ftz(A2 * base[q2] - c2) * d;
                }
                tb[kTabE1 + hs * kBlk + r] = ex2_ftz(c2 - A2 * own_base);   // row factor to the boundary
            } else {
                // 16-row sub-block of r: cs just before it and across it, in scan order
                const float half = __shfl_sync(MASK, s, dir > 0 ? 15 : 16);
                const bool second = dir > 0 ? lane >= 16 : lane < 16;
                const float pre2 = A2 * (own_base + (second ? half : 0.f));
                const float post2 = A2 * (own_base + (second ? own_tot : half));
                tb[kTabR16 + hs * kBlk + r] = ex2_ftz(c2 - pre2);
                tb[kTabD16 + hs * kBlk + r] = ex2_ftz(pre2 - c2) * d;
                tb[kTabO16 + hs * kBlk + r] = ex2_ftz(post2 - c2) * d;
                // the factorised sub-block is exact while its column factors stay far from
                // float32 overflow: decay across the sub-block below 2^-120
                if ((lane & 15) == 0) tb[kTabBig + hs * 8 + (r >> 4)] = (pre2 - post2 > 120.f) ? 1.f : 0.f;
                tb[kTabWR + hs * kBlk + r] = ex2_ftz(cl2 - c2) * d;
                tb[kTabER + hs * kBlk + r] = ex2_ftz(c2);
                if (r == 0) tb[kTabA + hs] = ex2_ftz(cl2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_TABREADY0 + sl));
            return true;
        };

        // w (.) x of block jj -> wX tile (same swizzled layout as the X tile), this half's 4 chunks
        auto wx_pass = [&](int jj) -> bool {
            const int st = jj & 1;
            if (!mbar_wait(bar(B_TABREADY0 + st), (jj >> 1) & 1, MASK, abort_flag, prm.status, 41)) return false;
            if (!mbar_wait(bar(B_XFULL0 + st), (jj >> 1) & 1, MASK, abort_flag, prm.status, 42)) return false;
            // w rounded to bf16 once, then one packed bf16 multiply per pair of x values
            const float wr = tab_s[st * kTabFloats + kTabWR + hs * kBlk + r];
            const uint32_t w2 = pack_bf16(wr, wr);
            const uint8_t *xt = sm + kOffX + st * kStageBytes + hs * kTileBytes;
#pragma unroll
            for (int qh = 0; qh < 2; ++qh) {
                float dx[16];                  // D x of 16 columns, the starting value of Y_diag
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = 4 * c + 2 * qh + qq;
                    const uint4 v = *reinterpret_cast<const uint4 *>(xt + swz(r, q));
                    uint4 o;
                    o.x = mul_bf16x2(v.x, w2);
                    o.y = mul_bf16x2(v.y, w2);
                    o.z = mul_bf16x2(v.z, w2);
                    o.w = mul_bf16x2(v.w, w2);
                    *reinterpret_cast<uint4 *>(wx_tile + swz(r, q)) = o;
                    const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        dx[8 * qq + 2 * i] = Dh * bf16lo(xw[i]);
                        dx[8 * qq + 2 * i + 1] = Dh * bf16hi(xw[i]);
                    }
                }
                tmem_st16f_nw(tl + colYD + 16 * qh, dx);
            }
            fence_async_smem();                // w(.)x is read by the tensor core
            tmem_wait_st();
            tc_fence_before();                 // Y_diag's starting value is read by the MMA
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_WXREADY));
            return true;
        };

        // state hand-off into block jj (>= 1): the state MMA of block jj - 1 has left S'
        // (entering block jj) in TMEM; thread r holds row n = r of this half's 32 columns.
        // bf16(S') goes to smem for Y_off = C S'^T, and S' is scaled in place by block jj's
        // decay so that block jj's state MMA accumulates S' <- exp(cs_last) S' + S directly.
        // state entering the scan (single direction with a carried state): S' of this row
        // (n = r) and half is read from global memory, a bf16 copy goes to smem for block 0's
        // Y_off and S' is scaled in place by block 0's decay, as the hand-off does between blocks
        const size_t sslot = ((size_t)b * prm.H + h) * kP * kN;   // [b][h] slot of s_in / s_out
        auto init_pass = [&]() {
            const float ablk = tab_s[kTabA + hs];
#pragma unroll 1
            for (int qd = 0; qd < 2; ++qd) {
                float sv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[i] = prm.s_in[sslot + (size_t)(32 * c + 16 * qd + i) * kN + r];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint4 o;
                    o.x = pack_bf16(sv[8 * qq + 0], sv[8 * qq + 1]);
                    o.y = pack_bf16(sv[8 * qq + 2], sv[8 * qq + 3]);
                    o.z = pack_bf16(sv[8 * qq + 4], sv[8 * qq + 5]);
                    o.w = pack_bf16(sv[8 * qq + 6], sv[8 * qq + 7]);
                    *reinterpret_cast<uint4 *>(sp_tile + swz(r, 4 * c + 2 * qd + qq)) = o;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[i] *= ablk;
                tmem_st16f_nw(tl + colST + 16 * qd, sv);
            }
            fence_async_smem();                // SP is read by the tensor core
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SPREADY));
        };

        auto state_pass = [&](int jj) {
            const float ablk = tab_s[(jj & 1) * kTabFloats + kTabA + hs];
            tc_fence_after();
#pragma unroll 1
            for (int qd = 0; qd < 2; ++qd) {
                float sv[16];
                tmem_ld16(tl + colST + 16 * qd, sv);
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint4 o;
                    o.x = pack_bf16(sv[8 * qq + 0], sv[8 * qq + 1]);
                    o.y = pack_bf16(sv[8 * qq + 2], sv[8 * qq + 3]);
                    o.z = pack_bf16(sv[8 * qq + 4], sv[8 * qq + 5]);
                    o.w = pack_bf16(sv[8 * qq + 6], sv[8 * qq + 7]);
                    *reinterpret_cast<uint4 *>(sp_tile + swz(r, 4 * c + 2 * qd + qq)) = o;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[i] *= ablk;
                tmem_st16f_nw(tl + colST + 16 * qd, sv);
            }
            fence_async_smem();                // SP is read by the tensor core
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SPREADY));
        };

        const int jend = (nblk > 0 && make_tables(0)) ? nblk : 0;
        for (int j = 0; j < jend; ++j) {
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            const int st = j & 1;
            const float *tb = tab_s + st * kTabFloats;
            if (!wx_pass(j)) break;
            if (j >= 1) {
                if (!mbar_wait(bar(B_STFULL), (j - 1) & 1, MASK, abort_flag, prm.status, 43)) break;
                state_pass(j);
            } else if (has_in) {
                init_pass();
            }

            // M_h = G (.) decay (.) dt over the causal triangle, bf16, for both heads.  This
            // warpgroup takes K-steps g and g + 4; the two heads' bf16 results for a K-step
            // replace the 16 float32 G columns they were computed from.
            if (!mbar_wait(bar(B_GFULL), j & 1, MASK, abort_flag, prm.status, 44)) break;
            tc_fence_after();
            {
                const float c2h[2] = {tb[kTabCS + r], tb[kTabCS + kBlk + r]};
                const float e1h[2] = {tb[kTabE1 + r], tb[kTabE1 + kBlk + r]};
#pragma unroll 1
                for (int ks = g; ks < 8; ks += 4) {
                    const int sq = ks >> 1;                          // source quarter
                    const bool offd = dir > 0 ? sq < wq : sq > wq;
                    const bool diag = sq == wq;
                    uint32_t m[16];
                    if (offd) {
                        float gv[16];
                        tmem_ld16(tl + kColG + 16 * ks, gv);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const float *wrow = tb + kTabW + (hh * 4 + wq) * kBlk + 16 * ks;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 wv = *reinterpret_cast<const float4 *>(wrow + 4 * i);
                                m[8 * hh + 2 * i] = pack_bf16(gv[4 * i] * wv.x * e1h[hh], gv[4 * i + 1] * wv.y * e1h[hh]);
                                m[8 * hh + 2 * i + 1] =
                                    pack_bf16(gv[4 * i + 2] * wv.z * e1h[hh], gv[4 * i + 3] * wv.w * e1h[hh]);
                            }
                        }
                    } else if (diag && tb[kTabBig + ks] == 0.f && tb[kTabBig + 8 + ks] == 0.f) {
                        // diagonal quarter, K-step = 16-row sub-block ks.  Row r's own sub-block:
                        // exp(cs_r - cs_s) = R16[r] D16[s] for s up to r in scan order; the
                        // sub-block before it in scan order: R16[r] O16[s]; the one after: 0.
                        float gv[16];
                        tmem_ld16(tl + kColG + 16 * ks, gv);
                        const int kt = r >> 4;
                        const bool own = kt == ks, prev = kt == ks + dir;
                        // keep source u (0..15 in the sub-block): u <= bound forward, u >= bound reverse
                        const int bound = own ? r - 16 * ks : prev ? (dir > 0 ? 15 : 0) : (dir > 0 ? -1 : 16);
                        bool keep[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u) keep[u] = dir > 0 ? u <= bound : u >= bound;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const float rf = tb[kTabR16 + hh * kBlk + r];
                            const float *crow = tb + (own ? kTabD16 : kTabO16) + hh * kBlk + 16 * ks;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 cv = *reinterpret_cast<const float4 *>(crow + 4 * i);
                                const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
                                float mv[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) mv[e] = keep[4 * i + e] ? gv[4 * i + e] * cc[e] * rf : 0.f;
                                m[8 * hh + 2 * i] = pack_bf16(mv[0], mv[1]);
                                m[8 * hh + 2 * i + 1] = pack_bf16(mv[2], mv[3]);
                            }
                        }
                    } else if (diag) {
                        // decay across the sub-block too steep for the factorised form: one
                        // exponential per element
                        float gv[16];
                        tmem_ld16(tl + kColG + 16 * ks, gv);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const float *csrc = tb + kTabCS + hh * kBlk + 16 * ks, *dsrc = tb + kTabDT + hh * kBlk + 16 * ks;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float4 cv = *reinterpret_cast<const float4 *>(csrc + 4 * i);
                                const float4 dv = *reinterpret_cast<const float4 *>(dsrc + 4 * i);
                                const float cc[4] = {cv.x, cv.y, cv.z, cv.w}, dd[4] = {dv.x, dv.y, dv.z, dv.w};
                                float mv[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int sidx = 16 * ks + 4 * i + e;
                                    const bool in = dir > 0 ? sidx <= r : sidx >= r;
                                    mv[e] = in ? gv[4 * i + e] * ex2_ftz(c2h[hh] - cc[e]) * dd[e] : 0.f;
                                }
                                m[8 * hh + 2 * i] = pack_bf16(mv[0], mv[1]);
                                m[8 * hh + 2 * i + 1] = pack_bf16(mv[2], mv[3]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) m[i] = 0u;       // outside the causal triangle
                    }
                    tmem_st16_nw(tl + kColG + 16 * ks, m);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_MREADY));

            // next block's decay tables, while the tensor core computes this block's Y_diag
            if (j + 1 < nblk && !make_tables(j + 1)) break;

            // epilogue: o = Y_diag (which started at D x) + exp(cs_r) Y_off, bf16, written over this row of the x
            // tile (free once the intra-block MMA is done); a store warp then writes the tile to y
            // in whole rows
            if (!mbar_wait(bar(hs == 0 ? B_YFULLH0 : B_YFULL), j & 1, MASK, abort_flag, prm.status, 46)) break;
            tc_fence_after();
            {
                uint8_t *xt = sm + kOffX + st * kStageBytes + hs * kTileBytes;
                float yv[32];
                if (j >= 1 || has_in) {
                    // Y_off of the incoming state, scaled by the decay exp(cs_r) up to this row
                    const float er = tb[kTabER + hs * kBlk + r];
                    float yo[32];
                    tmem_ld32x2(tl + colYD, tl + colYO, yv, yo);
#pragma unroll
                    for (int i = 0; i < 32; ++i) yv[i] = fmaf(er, yo[i], yv[i]);
                } else {
                    tmem_ld32(tl + colYD, yv);
                }
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int q = 4 * c + qq;
                    uint4 ov;
                    ov.x = pack_bf16(yv[8 * qq + 0], yv[8 * qq + 1]);
                    ov.y = pack_bf16(yv[8 * qq + 2], yv[8 * qq + 3]);
                    ov.z = pack_bf16(yv[8 * qq + 4], yv[8 * qq + 5]);
                    ov.w = pack_bf16(yv[8 * qq + 6], yv[8 * qq + 7]);
                    *reinterpret_cast<uint4 *>(xt + swz(r, q)) = ov;
                }
            }
            fence_async_smem();                // the tile is read by a TMA store
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_YEMPTY));
                mbar_arrive(bar(B_TILE00 + 2 * hs + st));
            }
            if (kState && j + 1 == nblk && prm.s_out) {
                // state leaving the scan: S' after the last block's state MMA, row n = r
                if (!mbar_wait(bar(B_STFULL), j & 1, MASK, abort_flag, prm.status, 49)) break;
                tc_fence_after();
#pragma unroll 1
                for (int qd = 0; qd < 2; ++qd) {
                    float sv[16];
                    tmem_ld16(tl + colST + 16 * qd, sv);
#pragma unroll
                    for (int i = 0; i < 16; ++i) prm.s_out[sslot + (size_t)(32 * c + 16 * qd + i) * kN + r] = sv[i];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// ------------------------------------------------------------------ host side

unsigned long long next_epoch() {
    // distinct per call in this process; the random start keeps a fresh workspace's
    // leftover contents from matching (flags are compared for equality)
    static std::atomic<unsigned long long> counter{
        0x9E3779B97F4A7C15ull ^ (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() ^
        ((unsigned long long)(uintptr_t)&counter << 17)};
    return counter.fetch_add(0x100000001ull) | 1ull;
}

}  // namespace

bool tc_supported(bool bf16, int batch, int L, int H, int P, int N, int G, int chunk) {
    return bf16 && P == kP && N == kN && G == 1 && H % 2 == 0 && H % 8 == 0 && chunk % kBlk == 0 &&
           L % kBlk == 0 && (long long)batch * L <= (1ll << 31) - 1 && get_encode() != nullptr;
}

namespace {
constexpr int kTargetCtas = 148;                      // one wave on a B200
}

int tc_segments(int batch, int L, int H) {
    // CTAs of a bidirectional call without segments: one per (batch row, head pair, direction)
    const long long units = (long long)batch * H;
    const int nblk = L / kBlk;
    if (units <= 0 || nblk < 4) return 1;
    long long k = kTargetCtas / units;
    if (k > nblk / 2) k = nblk / 2;
    if (k > 16) k = 16;
    if (k < 2) return 1;
    // no empty segment: the count that the segment length implies
    const int sb = (nblk + (int)k - 1) / (int)k;
    return (nblk + sb - 1) / sb;
}

int tc_segment_blocks(int L, int nseg) {
    const int nblk = L / kBlk;
    return nseg > 1 ? (nblk + nseg - 1) / nseg : nblk;
}

int tc_state_pieces(int batch, int L, int H, int nseg) {
    if (nseg <= 1) return 0;
    const int sb = tc_segment_blocks(L, nseg);
    const long long per_piece = (long long)batch * H * (nseg - 1);   // state CTAs per piece of a segment
    long long m = kTargetCtas / per_piece;
    if (m < 1) m = 1;
    if (m > sb) m = sb;
    const int pb = (sb + (int)m - 1) / (int)m;
    return (sb + pb - 1) / pb;                          // no empty piece
}

int tc_piece_blocks(int L, int nseg, int npiece) {
    const int sb = tc_segment_blocks(L, nseg);
    return npiece > 0 ? (sb + npiece - 1) / npiece : sb;
}

namespace {
size_t round256(size_t v) { return (v + 255) / 256 * 256; }
// Workspace: epoch-tagged ticket and ready words per (batch, head, block), the epoch-tagged steep
// marks per chain; with segments, the per-segment decays and local end states.
struct TcLayout {
    size_t ticket, ready, steep, ldec, sloc, total;
};
TcLayout tc_layout(int batch, int L, int H, int nseg) {
    const int npieces = nseg > 1 ? (nseg - 1) * tc_state_pieces(batch, L, H, nseg) : 0;
    TcLayout o{};
    const size_t nflags = (size_t)batch * H * (L / kBlk);
    o.ticket = 0;
    o.ready = nflags * 8;
    o.steep = round256(2 * nflags * 8);
    o.total = round256(o.steep + (size_t)batch * (H / 2) * 2 * 8);
    if (nseg > 1) {
        o.ldec = o.total;
        o.sloc = round256(o.ldec + (size_t)batch * H * 2 * npieces * 4);
        o.total = round256(o.sloc + (size_t)batch * H * 2 * npieces * kP * kN * 4);
    }
    return o;
}
}  // namespace

size_t tc_workspace_bytes(int batch, int L, int H, int, int nseg) { return tc_layout(batch, L, H, nseg).total; }

TcArgs make_tc_args(int batch, int L, int H, int chunk, void *ws, int *status) {
    TcArgs t{};
    t.batch = batch; t.L = L; t.H = H; t.chunk = chunk; t.ws = ws; t.status = status;
    t.nseg = tc_segments(batch, L, H);
    t.npiece = tc_state_pieces(batch, L, H, t.nseg);
    t.concurrent = true;
    return t;
}

void tc_set_direction(TcArgs &t, int slot, int dir, const void *x, const void *dt, const float *A, const void *B,
                      const void *C, const float *D) {
    t.d[slot] = TcDir{x, dt, B, C, A, D, dir};
}

// Every call runs the shared-score kernel and then the exact kernel for the chains it left
// (which returns at once when there are none); a segmented call runs the segment-state kernel
// first.
int tc_launches(bool, int) { return 3; }   // steep marks (or segment states), scan, exact kernel

namespace {
// Steep-decay marks of a whole-sequence call (a segmented call's state kernel makes them): for
// each chain (batch row, head pair, direction) with a 128-token block whose decay passes
// kSteepLog2 for either head (log2 units, or is not a number), marks[(b H/2 + pair) 2 + slot] =
// epoch.  Nothing else decides which kernel runs a chain of the call, so the shared-score kernel
// and the exact kernel agree by construction.  One CTA per (block, batch row, direction), one
// thread per token: the thread reads its token's whole dt row (16-byte loads, so each row is
// read once for all heads), a warp butterfly sums 8 heads at a time, the 4 warps' sums meet
// in shared memory.
struct SteepArgs {
    const __nv_bfloat16 *dt[2];
    const float *A[2];
    unsigned long long *marks;
    unsigned long long epoch;
    int L, H;
};

__global__ void __launch_bounds__(128) k_ssd_steep_marks(const __grid_constant__ SteepArgs a) {
    extern __shared__ float part[];                     // [4 warps][H] per-warp sums
    const int blk = blockIdx.x, b = blockIdx.y, slot = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = (size_t)b * a.L + (size_t)blk * kBlk + threadIdx.x;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.dt[slot] + row * a.H);
    const int ng = a.H / 8;
    for (int g0 = 0; g0 < ng; g0 += 8) {
        uint4 v[8];                                     // up to eight groups of 8 heads in flight
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (g0 + i < ng) v[i] = src[g0 + i];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (g0 + i >= ng) break;
            const float d[8] = {bf16lo(v[i].x), bf16hi(v[i].x), bf16lo(v[i].y), bf16hi(v[i].y),
                                bf16lo(v[i].z), bf16hi(v[i].z), bf16lo(v[i].w), bf16hi(v[i].w)};
            // Sums over the warp's 32 rows by a reduce-scatter butterfly: each level hands the
            // partner lane the half of the heads it keeps and adds the half it receives, so lane l
            // ends with the sum of head (l >> 2) & 7 (9 shuffles for the 8 heads).
            const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
            float e4[4], e2[2];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                e4[k] = (b4 ? d[k + 4] : d[k]) + __shfl_xor_sync(0xffffffffu, b4 ? d[k] : d[k + 4], 16);
#pragma unroll
            for (int k = 0; k < 2; ++k)
                e2[k] = (b3 ? e4[k + 2] : e4[k]) + __shfl_xor_sync(0xffffffffu, b3 ? e4[k] : e4[k + 2], 8);
            float e1 = (b2 ? e2[1] : e2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? e2[0] : e2[1], 4);
            e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
            e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
            if ((lane & 3) == 0) part[warp * a.H + 8 * (g0 + i) + ((lane >> 2) & 7)] = e1;
        }
    }
    __syncthreads();
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
        const float sum = (part[h] + part[a.H + h]) + (part[2 * a.H + h] + part[3 * a.H + h]);
        const float ah = fabsf(a.A[slot][h]) * 1.4426950408889634f;
        if (ah * sum > kSteepLog2 || !(sum == sum))
            *reinterpret_cast<volatile unsigned long long *>(a.marks + ((size_t)b * (a.H / 2) + h / 2) * 2 + slot) =
                a.epoch;
    }
}

cudaError_t launch_steep_marks(const TcArgs &t, bool bidir, unsigned long long *marks, unsigned long long epoch,
                               cudaStream_t st) {
    SteepArgs a{};
    for (int s = 0; s < (bidir ? 2 : 1); ++s) {
        a.dt[s] = static_cast<const __nv_bfloat16 *>(t.d[s].dt);
        a.A[s] = t.d[s].A;
    }
    a.marks = marks;
    a.epoch = epoch;
    a.L = t.L;
    a.H = t.H;
    dim3 grid((unsigned)(t.L / kBlk), (unsigned)t.batch, bidir ? 2u : 1u);
    k_ssd_steep_marks<<<grid, kBlk, 4 * t.H * (int)sizeof(float), st>>>(a);
    return cudaGetLastError();
}
}  // namespace



cudaError_t launch_tc(const TcArgs &t, bool bidir, void *y, cudaStream_t st) {
    const int nseg = t.nseg > 1 ? t.nseg : 1;
    const TcLayout lo = tc_layout(t.batch, t.L, t.H, nseg);
    char *ws = static_cast<char *>(t.ws);
    unsigned long long *ticket = reinterpret_cast<unsigned long long *>(ws + lo.ticket);
    unsigned long long *ready = reinterpret_cast<unsigned long long *>(ws + lo.ready);
    SegScratch sc{};
    sc.steep = reinterpret_cast<unsigned long long *>(ws + lo.steep);
    if (nseg > 1) {
        sc.sloc = reinterpret_cast<float *>(ws + lo.sloc);
        sc.ldec = reinterpret_cast<float *>(ws + lo.ldec);
    }
    const unsigned long long epoch = next_epoch();
    const bool with_state = !bidir && (t.s_in || t.s_out);
    // The shared-memory opt-in belongs to the kernel in the current context: set on every launch.
    cudaError_t e =
        cudaFuncSetAttribute(with_state ? k_ssd_tc<true> : k_ssd_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int ndir = bidir ? 2 : 1;
    const uint64_t rows = (uint64_t)t.batch * t.L;
    TcMaps maps;
    memset(&maps, 0, sizeof maps);
    TcParams p{};
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
    p.bidir = bidir ? 1 : 0;
    p.dir_single = t.d[0].dir;
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.status = t.status;
    p.ticket = ticket;
    p.ready = ready;
    p.epoch = epoch;
    p.wait_cycles = t.wait_cycles;
    p.fault = t.fault;
    p.s_in = bidir ? nullptr : t.s_in;
    p.s_out = bidir ? nullptr : t.s_out;
    const int grid = t.batch * (t.H / 2) * ndir;
    p.steep = sc.steep;
    // the steep marks: the state kernel makes them for a segmented call, one pass otherwise
    if (nseg > 1) {
        if ((e = launch_segstate(t, bidir, sc, epoch, st)) != cudaSuccess) return e;
    } else if ((e = launch_steep_marks(t, bidir, sc.steep, epoch, st)) != cudaSuccess) {
        return e;
    }
    if ((e = launch_tcs(t, bidir, y, ticket, ready, sc, epoch, st)) != cudaSuccess) return e;
    // The exact kernel may start while the shared-score kernel still runs (programmatic
    // dependent launch: that kernel lets its dependents go as each CTA starts), so the steep
    // chains, each one long single-CTA walk, overlap the rest of the call.  Its last CTA only
    // waits for the shared-score grid to complete, so that work queued after this call sees
    // both kernels done.
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(grid + 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    if (t.concurrent) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return with_state ? cudaLaunchKernelEx(&cfg, k_ssd_tc<true>, maps, p)
                      : cudaLaunchKernelEx(&cfg, k_ssd_tc<false>, maps, p);
}

}  // namespace ssd
