// ssd_tcs_seg.cu -- local end states of sequence segments, for the shared-score
// scan run over segments of a sequence in parallel.
//
// A chain (batch row, head, direction) of nblk 128-token blocks is cut into
// nseg segments of consecutive blocks in scan order.  The recurrence
// S <- exp(dt A) S + dt x (outer) B is linear in S, so the state entering
// segment s is
//
//   S_in(s) = exp(A T_{s-1}) S_in(s-1) + S_loc(s-1),   S_in(0) = the state entering the scan,
//
// with T_s the sum of dt over segment s and S_loc(s) the state segment s leaves
// when it starts from zero:
//
//   S_loc(s) = sum_{i in s} exp(A (T_end - T_i)) dt_i x_i (outer) B_i,
//
// T_i the running sum of dt in scan order ("Mamba-2 / SSD" state-passing form,
// as the DiffuMamba technical summary's bidirectional layers run it, section 2).
// Every weight w_i = exp(A (T_end - T_i)) dt_i lies in [0, dt_i]: walking the
// segment's blocks from its end backwards, the suffix sum of dt is known when a
// block is reached, so one accumulator sums B^T (w x) over the whole segment on
// the tensor core with no rescaling and nothing that can overflow.
//
// Each segment but the last (nothing needs the last one's local state) is
// formed in npiece pieces of consecutive blocks, so that the kernel has about
// as many CTAs as the GPU has SMs: one CTA per (batch row, head pair,
// direction, piece).  The scan folds the pieces in order.  The CTAs also run
// the steep-decay test (steep_of_block, the one the other kernels use) on
// every block of the chain, their own pieces' blocks from the dt tiles they
// load and a share of the last segment's from global memory, and mark the
// chain steep in the workspace: the scan and the exact kernel then agree on
// which chains the exact kernel takes.
//
// Warps (576 threads): warp 0 loads x, B and dt (TMA) into three stages; warp 1
// owns TMEM and issues the MMAs; warps 2-17 weight the rows of x in place
// (warp 2 + 8 hs + 2 q + c: head hs, rows 32 q .. 32 q + 31, 16-byte chunks
// 4 c .. 4 c + 3) and read the result out.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "ssd_tc.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kBlk = 128, kP = 64, kN = 128;
constexpr int kThreads = 576;
constexpr int kCw = 16;                                 // weighting warps
constexpr int kStages = 3;
constexpr uint32_t kTileBytes = kBlk * 64 * 2;          // [128][64] bf16, 128-byte swizzled
constexpr uint32_t kPairBytes = 2 * kTileBytes;
constexpr uint32_t kDtBytes = kBlk * 8 * 2;             // dt box: 128 tokens x 8 heads
// stage: x (two heads) | B (two n halves) | dt
constexpr uint32_t kStX = 0, kStB = kPairBytes, kStDt = 2 * kPairBytes;
constexpr uint32_t kStageBytes = (2 * kPairBytes + kDtBytes + 1023) / 1024 * 1024;
constexpr uint32_t kOffTab = kStages * kStageBytes;     // per stage and head: w of the block's 128 rows
constexpr uint32_t kOffBar = kOffTab + kStages * 2 * kBlk * 4;
enum Bar { B_FULL0 = 0, B_EMPTY0 = B_FULL0 + kStages, B_WREADY0 = B_EMPTY0 + kStages,
           B_TAB0 = B_WREADY0 + kStages,                // [stage][head]
           B_DONE = B_TAB0 + 2 * kStages, kNumBars };
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem slot, abort flag, wait limit
constexpr uint32_t kSmemBytes = kOffMisc + 32 + 1024;
static_assert(kStageBytes % 1024 == 0 && kSmemBytes <= 232448, "shared memory layout");
constexpr float kLog2e = 1.4426950408889634f;

struct SegParams {
    int batch, L, H, nblk, nseg, sb, npiece, pb, bidir, dir_single;
    const float *A[2];
    const __nv_bfloat16 *dt[2];
    float *sloc;                        // [batch][H][2][(nseg - 1) npiece][P][N]
    float *ldec;                        // [batch][H][2][(nseg - 1) npiece]: A T over the piece, log2 units
    unsigned long long *steep;          // [batch][H/2][2], epoch-tagged
    unsigned long long epoch;
    int *status;
    long long wait_cycles;
};
struct SegMaps {
    CUtensorMap x[2], dt[2], b[2];
};

__global__ void __launch_bounds__(kThreads, 1) k_ssd_segstate(const __grid_constant__ SegMaps maps,
                                                              const __grid_constant__ SegParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);   // limit at +8

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = prm.bidir ? (blockIdx.x & 1) : 0;
    const int dir = prm.bidir ? (slot == 0 ? 1 : -1) : prm.dir_single;
    const int unit = prm.bidir ? (blockIdx.x >> 1) : blockIdx.x;
    const int npieces = (prm.nseg - 1) * prm.npiece;   // pieces of a chain
    const int piece = unit % npieces, pu = unit / npieces;
    const int npairs = prm.H / 2;
    const int b = pu / npairs, hp = pu % npairs, h0 = 2 * hp;
    const int nblk = prm.nblk, L = prm.L;
    // this piece: scan-order blocks g0 .. g0 + nb - 1 of segment piece / npiece
    const int g0 = (piece / prm.npiece) * prm.sb + (piece % prm.npiece) * prm.pb;
    const int nb = min(prm.pb, (piece / prm.npiece + 1) * prm.sb - g0);
    // memory block of scan block g
    auto mblk = [&](int g) { return dir > 0 ? g : nblk - 1 - g; };
    const float a0 = fabsf(prm.A[slot][h0]) * kLog2e, a1 = fabsf(prm.A[slot][h0 + 1]) * kLog2e;
    unsigned long long *steep_mark = prm.steep + ((size_t)b * npairs + hp) * 2 + slot;

    // steep-decay test of this CTA's share of the last segment's blocks (the pieces' own blocks
    // are tested from their dt tiles below)
    if (warp >= 2) {
        bool steep = false;
        for (int g = (prm.nseg - 1) * prm.sb + piece + npieces * (warp - 2); g < nblk; g += npieces * kCw)
            steep |= block_is_steep(prm.dt[slot], a0, a1, b, L, prm.H, h0, mblk(g), lane);
        if (steep && lane == 0) *reinterpret_cast<volatile unsigned long long *>(steep_mark) = prm.epoch;
    }
    if (nb <= 0) return;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < (int)kNumBars; ++i)
            mbar_init(bar(i), (i >= B_WREADY0 && i < B_WREADY0 + kStages) ? kCw : 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t MASK = 0xffffffffu;

    if (warp == 0) {
        // ---------------------------------------------------------- loads, last block first
        int issued = 0;
        if (lane == 0) {
            for (int i = 0; i < nb; ++i) {
                const int st = i % kStages;
                if (i >= kStages &&
                    !mbar_wait(bar(B_EMPTY0 + st), ((i / kStages) - 1) & 1, 1u, abort_flag, prm.status, 81))
                    break;
                const int row = b * L + mblk(g0 + nb - 1 - i) * kBlk;
                const uint32_t base = sbase + st * kStageBytes;
                mbar_expect_tx(bar(B_FULL0 + st), 2 * kPairBytes + kDtBytes);
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(base + kStX + h * kTileBytes, &maps.x[slot], (h0 + h) * kP, row, bar(B_FULL0 + st));
                for (int q = 0; q < 2; ++q)
                    tma_load_2d(base + kStB + q * kTileBytes, &maps.b[slot], q * 64, row, bar(B_FULL0 + st));
                tma_load_2d(base + kStDt, &maps.dt[slot], h0 & ~7, row, bar(B_FULL0 + st));
                issued = i + 1;
            }
            if (*abort_flag) {
                for (int i = issued - 1; i >= 0 && i >= issued - kStages; --i)
                    mbar_drain(bar(B_FULL0 + i % kStages), (i / kStages) & 1, prm.wait_cycles);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- S += B^T (w x): M = n, N = (head, p), K = rows
        const uint32_t id_s = idesc(128, 1, 1);
        for (int i = 0; i < nb; ++i) {
            const int st = i % kStages;
            if (!mbar_wait(bar(B_FULL0 + st), (i / kStages) & 1, MASK, abort_flag, prm.status, 82)) break;
            if (!mbar_wait(bar(B_WREADY0 + st), (i / kStages) & 1, MASK, abort_flag, prm.status, 83)) break;
            tc_fence_after();
            const uint32_t base = sbase + st * kStageBytes;
            const SDesc dBm = make_sdesc(base + kStB, kTileBytes, 1024), dX = make_sdesc(base + kStX, kTileBytes, 1024);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) mma_ss_w(tmem, dBm.at(ks * 2048), dX.at(ks * 2048), id_s, (i > 0) || (ks > 0));
            mma_commit_w(bar(B_EMPTY0 + st));
        }
        mma_commit_w(bar(B_DONE));                       // every MMA issued has completed
        if (lane == 0) mbar_drain(bar(B_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // ---------------------------------------------------------- weights w, rows of x scaled in place
        const int cw = warp - 2, hs = cw >> 3, q = (cw >> 1) & 3, c4 = cw & 1;
        const int h = h0 + hs;
        const float A2 = prm.A[slot][h] * kLog2e;        // log2 units, <= 0
        // the weights of a block live with its stage: rewritten only once its stage is reloaded,
        // after every warp has passed the block (B_WREADY, then the MMA, then B_EMPTY)
        float *tabs = reinterpret_cast<float *>(sm + kOffTab) + hs * kBlk;
        float carry = 0.f;                               // sum of dt over the piece's blocks after this one
        bool ok = true, steep = false;
        for (int i = 0; i < nb && ok; ++i) {
            const int st = i % kStages;
            if (!mbar_wait(bar(B_FULL0 + st), (i / kStages) & 1, MASK, abort_flag, prm.status, 84)) {
                ok = false;
                break;
            }
            uint8_t *base = sm + st * kStageBytes;
            const uint8_t *dtt = base + kStDt;           // [128 rows][8 heads] bf16
            if (i % kCw == cw) {
                // the steep test of this block, from the tile: row lane + 32 i of the block
                uint32_t u[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    u[e] = *reinterpret_cast<const uint32_t *>(dtt + (lane + 32 * e) * 16 + (h0 & 7) * 2);
                steep |= steep_of_block(u, a0, a1);
            }
            float *tab = tabs + st * 2 * kBlk;
            // one warp per head (rows 0-31, chunks 0-3) builds the head's weights: lane l holds
            // scan positions l + 32 t (memory row k forward, 127 - k reverse); the suffix sum
            // of position k is the later columns' totals plus the later lanes of its column
            if ((cw & 7) == 0) {
                float d[4];
                int rows[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int k = lane + 32 * t;
                    rows[t] = dir > 0 ? k : kBlk - 1 - k;
                    d[t] = __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16 *>(dtt + rows[t] * 16 + ((h0 & 7) + hs) * 2));
                }
                float incl[4], col[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    incl[t] = d[t];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float u = __shfl_up_sync(MASK, incl[t], o);
                        if (lane >= o) incl[t] += u;
                    }
                    col[t] = __shfl_sync(MASK, incl[t], 31);
                }
                float later = carry;                     // dt of the columns after t, and of the blocks after
#pragma unroll
                for (int t = 3; t >= 0; --t) {
                    tab[rows[t]] = ex2_ftz(A2 * (later + col[t] - incl[t])) * d[t];
                    later += col[t];
                }
                carry = later;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_TAB0 + 2 * st + hs));
            } else if (!mbar_wait(bar(B_TAB0 + 2 * st + hs), (i / kStages) & 1, MASK, abort_flag, prm.status, 86)) {
                ok = false;
                break;
            }
            // this warp's rows and chunks of its head's x tile, scaled by w in place (fp32 multiply,
            // one rounding)
            const int r = q * 32 + lane;
            const float w = tab[r];
            uint8_t *xt = base + kStX + hs * kTileBytes;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int c = 4 * c4 + cc;
                const uint4 v = *reinterpret_cast<const uint4 *>(xt + swz(r, c));
                const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) o[e] = pack_bf16(bf16lo(xw[e]) * w, bf16hi(xw[e]) * w);
                *reinterpret_cast<uint4 *>(xt + swz(r, c)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_async_smem();                          // read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_WREADY0 + st));
        }
        if (steep && lane == 0) *reinterpret_cast<volatile unsigned long long *>(steep_mark) = prm.epoch;
        // read out: TMEM lane quarter warp % 4 (rows n), 32 columns of group cw >> 2 (head, p half)
        if (ok && mbar_wait(bar(B_DONE), 0, MASK, abort_flag, prm.status, 85)) {
            tc_fence_after();
            const int n = (warp & 3) * 32 + lane, cg = cw >> 2;
            const int ho = cg >> 1, p0 = (cg & 1) * 32;
            float v[32];
            tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 32 * cg, v);
            const size_t chain = ((size_t)b * prm.H + h0 + ho) * 2 + slot;
            float *out = prm.sloc + (chain * npieces + piece) * kP * kN;
#pragma unroll
            for (int p = 0; p < 32; ++p) out[(size_t)(p0 + p) * kN + n] = v[p];
            if ((cw & 7) == 0 && lane == 0) prm.ldec[(((size_t)b * prm.H + h) * 2 + slot) * npieces + piece] = A2 * carry;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
    }
}

}  // namespace

cudaError_t launch_segstate(const TcArgs &t, bool bidir, const SegScratch &sc, unsigned long long epoch,
                            cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(k_ssd_segstate, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int ndir = bidir ? 2 : 1;
    const uint64_t rows = (uint64_t)t.batch * t.L;
    SegMaps maps;
    memset(&maps, 0, sizeof maps);
    SegParams p{};
    for (int s = 0; s < ndir; ++s) {
        const TcDir &d = t.d[s];
        if (!make_map(&maps.x[s], d.x, rows, (uint64_t)t.H * kP, 64, true) ||
            !make_map(&maps.dt[s], d.dt, rows, (uint64_t)t.H, 8, false) ||
            !make_map(&maps.b[s], d.B, rows, kN, 64, true))
            return cudaErrorInvalidValue;
        p.A[s] = d.A;
        p.dt[s] = static_cast<const __nv_bfloat16 *>(d.dt);
    }
    p.batch = t.batch; p.L = t.L; p.H = t.H; p.nblk = t.L / kBlk;
    p.nseg = t.nseg; p.sb = tc_segment_blocks(t.L, t.nseg);
    p.npiece = t.npiece; p.pb = tc_piece_blocks(t.L, t.nseg, t.npiece);
    p.bidir = bidir ? 1 : 0;
    p.dir_single = t.d[0].dir;
    p.sloc = sc.sloc; p.ldec = sc.ldec; p.steep = sc.steep;
    p.epoch = epoch;
    p.status = t.status;
    p.wait_cycles = t.wait_cycles;
    const int grid = t.batch * (t.H / 2) * (t.nseg - 1) * t.npiece * ndir;
    k_ssd_segstate<<<grid, kThreads, kSmemBytes, st>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace ssd
