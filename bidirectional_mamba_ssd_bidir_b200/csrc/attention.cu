// Multi-head softmax attention without a mask, on the tensor core (tcgen05, TMEM, TMA).
//
// "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", technical
// summary, section 2: DiffuMamba-H puts one Transformer block (an attention
// mixer) after every five Mamba blocks.  The page leaves the attention itself
// open; it is read as the attention of a diffusion language model, every token
// seeing the whole sequence:
//
//   O[b, i, h] = sum_j softmax_j(scale q[b, i, h] . k[b, j, h]) v[b, j, h]
//
// One CTA per (two tiles of 128 queries, head, sequence), walking the keys in tiles of 128.
// For each query tile t and key tile j:
//
//   S_t  = Q_t K_j^T               SS MMA into TMEM
//   P_t  = 2^(S_t c - m)           CUDA cores, one thread per query row; bf16, written over
//                                  S_t in TMEM (c = scale log2 e)
//   O_t += P_t V_j                 TS MMA: A = P from TMEM, B = V (MN-major) from shared memory
//
// The two query tiles share each K/V tile and take turns: while one tile's softmax warps work,
// the tensor core runs the other tile's products (TMEM: S_0, O_0, S_1, O_1, 128 columns each).
// The reference m of a row follows the row maximum lazily: it moves only when a tile's maximum
// exceeds it by more than 8 (log2 units), so p <= 2^8 and O (in TMEM) is rescaled by 2^(m_old
// - m_new) only on those tiles.  The row sum l accumulates p (float32); the epilogue writes
// O / l.  Tiles reach past the sequence's end as zeros (3-D tensor
// maps clip at each sequence); those keys are masked to p = 0 and those query rows are not
// stored.
//
// Warps (320 threads): warp 0 issues the TMA loads, warp 1 owns TMEM and issues the MMAs, warps
// 2-5 run query tile 0's softmax and epilogue, warps 6-9 tile 1's (TMEM lane quarter warp % 4).
// Every wait is bounded; a wait that runs out records its code in the status word and the CTA
// winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "attention.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kAQ = 128;                       // query rows per tile (= TMEM lanes)
constexpr int kATiles = 2;                     // query tiles per CTA
constexpr int kAKeys = 128;                    // keys per tile
constexpr int kAThreads = 64 + kATiles * 128;
constexpr int kAStages = 2;                    // K/V tiles in flight
constexpr uint32_t kABox = 128 * 128;          // one [128 rows][64 bf16] swizzled box: 16 KB

enum AttnBar {
    AB_QFULL = 0,
    AB_KFULL0,
    AB_VFULL0 = AB_KFULL0 + kAStages,
    AB_KVEMPTY0 = AB_VFULL0 + kAStages,
    AB_SFULL0 = AB_KVEMPTY0 + kAStages,        // per query tile
    AB_PREADY0 = AB_SFULL0 + kATiles,
    AB_ODONE0 = AB_PREADY0 + kATiles,
    AB_OSTAGED0 = AB_ODONE0 + kATiles,
    AB_DONE = AB_OSTAGED0 + kATiles,
    kAttnBars
};

template <int D>
struct AttnLayout {
    static constexpr uint32_t kTile = (D / 64) * kABox;          // a [128][D] tile
    static constexpr uint32_t kOffQ = 0;                         // Q_t at t kTile; O_t there at the end
    static constexpr uint32_t kOffKV = kATiles * kTile;          // stage s: K at + 2 s kTile, V after it
    static constexpr uint32_t kOffBar = kOffKV + kAStages * 2 * kTile;
    static constexpr uint32_t kOffMisc = kOffBar + kAttnBars * 8;   // tmem base, abort flag, wait limit
    // + alignment slack; at least 116 KB, so that one CTA fits per SM (each holds all 512 TMEM
    // columns: a second one would only wait in its allocation)
    static constexpr uint32_t kSmemNeed = kOffMisc + 16 + 1024;
    static constexpr uint32_t kSmem = kSmemNeed > 116u * 1024 ? kSmemNeed : 116u * 1024;
};

struct AttnMaps {
    CUtensorMap q, k, v, o;
};
struct AttnParams {
    int L, ntiles;
    float scale_log2;
    int *status;
    long long wait_cycles;
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// Optional hand-off timeline for the tracing build (-DSSD_TRACE): SM-clock stamps of CTA 0 for
// its first kATraceTiles key tiles, [point][tile]: 0/1 PV_t issued (t = 0, 1), 2/3 S_t(j + 1)
// issued, 4/5 the softmax of tile t started (its S arrived; warp of lane quarter 2), 6/7 that
// warp handed its P over.
#ifdef SSD_TRACE
constexpr int kATraceTiles = 32, kATracePts = 8;
__device__ unsigned long long g_attn_trace[kATracePts * kATraceTiles];
__device__ __forceinline__ void attn_pt(int k, int j) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && j < kATraceTiles && (threadIdx.x & 31) == 0)
        g_attn_trace[k * kATraceTiles + j] = clock64();
}
#define ATTN_PT(k, j) attn_pt(k, j)
#else
#define ATTN_PT(k, j) ((void)0)
#endif

template <int D>
__global__ void __launch_bounds__(kAThreads, 1) k_attention(const __grid_constant__ AttnMaps maps,
                                                            const __grid_constant__ AttnParams prm) {
    using Lo = AttnLayout<D>;
    constexpr int kBoxes = D / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + Lo::kOffBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lo::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lo::kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * (kATiles * kAQ), hcol = blockIdx.y * D, b = blockIdx.z;
    const int nt = prm.ntiles;
    const uint32_t MASK = 0xffffffffu;
    auto col_s = [](int t) { return 256u * t; };             // TMEM columns of S_t (P_t over it)
    auto col_o = [](int t) { return 256u * t + 128u; };      // and of O_t

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kAttnBars; ++i) {
            const bool four = (i >= AB_PREADY0 && i < AB_PREADY0 + kATiles) ||
                              (i >= AB_OSTAGED0 && i < AB_OSTAGED0 + kATiles);
            mbar_init(bar(i), four ? 4u : 1u);
        }
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
        // ------------------------------------------------------------ TMA loads
        if (lane == 0) {
            mbar_expect_tx(bar(AB_QFULL), kATiles * Lo::kTile);
            for (int t = 0; t < kATiles; ++t)
                for (int x = 0; x < kBoxes; ++x)
                    tma_load_3d(sbase + Lo::kOffQ + t * Lo::kTile + x * kABox, &maps.q, hcol + 64 * x, q0 + kAQ * t,
                                b, bar(AB_QFULL));
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int s = j % kAStages;
                // the stage is free once both PV products of tile j - kAStages have completed
                if (j >= kAStages &&
                    !mbar_wait(bar(AB_KVEMPTY0 + s), ((j / kAStages) - 1) & 1, 1u, abort_flag, prm.status, 131))
                    break;
                const uint32_t kb = sbase + Lo::kOffKV + s * 2 * Lo::kTile, vb = kb + Lo::kTile;
                mbar_expect_tx(bar(AB_KFULL0 + s), Lo::kTile);
                for (int x = 0; x < kBoxes; ++x)
                    tma_load_3d(kb + x * kABox, &maps.k, hcol + 64 * x, j * kAKeys, b, bar(AB_KFULL0 + s));
                mbar_expect_tx(bar(AB_VFULL0 + s), Lo::kTile);
                for (int x = 0; x < kBoxes; ++x)
                    tma_load_3d(vb + x * kABox, &maps.v, hcol + 64 * x, j * kAKeys, b, bar(AB_VFULL0 + s));
                issued = j + 1;
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA gives up its shared memory
                mbar_drain(bar(AB_QFULL), 0, prm.wait_cycles);
                for (int j = issued - 1; j >= 0 && j >= issued - kAStages; --j) {
                    mbar_drain(bar(AB_KFULL0 + j % kAStages), (j / kAStages) & 1, prm.wait_cycles);
                    mbar_drain(bar(AB_VFULL0 + j % kAStages), (j / kAStages) & 1, prm.wait_cycles);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMAs (one elected lane)
        // Order per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1); S_t(j+1) is written over
        // P_t(j), so it waits for PV_t(j) to complete.
        const uint32_t id_s = idesc(128, 0, 0);    // S = Q K^T: M = queries, N = keys, K = d
        const uint32_t id_o = idesc(D, 0, 1);      // O += P V: M = queries, N = d, K = keys
        // Q and K K-major (rows of 128 bytes, 8-row groups 1 KB apart, 64-column boxes kABox
        // apart); V MN-major (64-column chunks kABox apart, 8-key groups 1 KB apart)
        auto issue_s = [&](int t, int j) {
            const SDesc dq = make_sdesc(sbase + Lo::kOffQ + t * Lo::kTile, 16, 1024);
            const SDesc dk = make_sdesc(sbase + Lo::kOffKV + (j % kAStages) * 2 * Lo::kTile, 16, 1024);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (ks >> 2) * kABox + (ks & 3) * 32;
                mma_ss_w(tmem + col_s(t), dq.at(off), dk.at(off), id_s, ks > 0);
            }
            mma_commit_w(bar(AB_SFULL0 + t));
        };
        bool ok = mbar_wait(bar(AB_QFULL), 0, MASK, abort_flag, prm.status, 132) &&
                  mbar_wait(bar(AB_KFULL0), 0, MASK, abort_flag, prm.status, 133);
        if (ok) {
            tc_fence_after();
            for (int t = 0; t < kATiles; ++t) issue_s(t, 0);
        }
        for (int j = 0; j < nt && ok; ++j) {
            const int s = j % kAStages, s1 = (j + 1) % kAStages;
            if (!(ok = mbar_wait(bar(AB_VFULL0 + s), (j / kAStages) & 1, MASK, abort_flag, prm.status, 134))) break;
            const SDesc dv = make_sdesc(sbase + Lo::kOffKV + s * 2 * Lo::kTile + Lo::kTile, kABox, 1024);
            for (int t = 0; t < kATiles && ok; ++t) {
                // PV_t(j) once tile t's P is ready, then S_t(j + 1) over it once PV_t(j) has
                // completed: the tensor core runs tile t's products while the other tile is in
                // its softmax
                if (!(ok = mbar_wait(bar(AB_PREADY0 + t), j & 1, MASK, abort_flag, prm.status, 135))) break;
                tc_fence_after();
                // A = P_t (keys 16 ks .. 16 ks + 15 at TMEM columns [16 ks, 16 ks + 8) of S_t)
#pragma unroll
                for (int ks = 0; ks < kAKeys / 16; ++ks)
                    mma_ts_w(tmem + col_o(t), tmem + col_s(t) + 16 * ks, dv.at(ks * 2048), id_o, (j | ks) != 0);
                mma_commit_w(bar(AB_ODONE0 + t));
                ATTN_PT(t, j);
                if (t == kATiles - 1) mma_commit_w(bar(AB_KVEMPTY0 + s));
                if (j + 1 < nt) {
                    if (!(ok = mbar_wait(bar(AB_KFULL0 + s1), ((j + 1) / kAStages) & 1, MASK, abort_flag, prm.status,
                                         136)))
                        break;
                    if (!(ok = mbar_wait(bar(AB_ODONE0 + t), j & 1, MASK, abort_flag, prm.status, 137))) break;
                    tc_fence_after();
                    issue_s(t, j + 1);
                    ATTN_PT(2 + t, j);
                }
            }
        }
        // every MMA issued has completed before TMEM is released
        mma_commit_w(bar(AB_DONE));
        if (lane == 0) mbar_drain(bar(AB_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax, epilogue
        const int t = (warp - 2) >> 2;                            // query tile
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;                        // query row in the tile = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
        const uint32_t cs = col_s(t), co = col_o(t);
        float m_ref = 0.f, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            if (!(ok = mbar_wait(bar(AB_SFULL0 + t), j & 1, MASK, abort_flag, prm.status, 138))) break;
            if (quarter == 2) ATTN_PT(4 + t, j);
            tc_fence_after();
            float x[128];
            tmem_ld32x2(tl + cs, tl + cs + 32, x, x + 32);
            tmem_ld32x2(tl + cs + 64, tl + cs + 96, x + 64, x + 96);
            const int valid = prm.L - j * kAKeys;               // keys of this tile inside the sequence
            if (valid < kAKeys) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i >= valid) x[i] = -INFINITY;
            }
            // row maximum of the raw scores: eight independent chains (scale > 0 commutes with max)
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = x[i];
#pragma unroll
            for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], x[i]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * prm.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (j == 0) {
                m_ref = mx;                                     // tile 0 holds at least one key
            } else {
                const bool need = mx > m_ref + 8.f;
                if (need) {
                    alpha = ex2_ftz(m_ref - mx);
                    m_ref = mx;
                }
                rescale = __any_sync(MASK, need);
            }
            // P = 2^(x c - m_ref) as bf16 over S (one packed FMA per pair for the argument); the
            // row sum in four independent packed chains
            const float2 c2 = make_float2(prm.scale_log2, prm.scale_log2), nm2 = make_float2(-m_ref, -m_ref);
            float2 acc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t pw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 a = fma2(make_float2(x[16 * ks + 2 * i], x[16 * ks + 2 * i + 1]), c2, nm2);
                    const float2 p2 = make_float2(ex2_ftz(a.x), ex2_ftz(a.y));
                    pw[i] = pack_bf16(p2.x, p2.y);
                    acc[i & 3] = add2(acc[i & 3], p2);
                }
                tmem_st8_nw(tl + cs + 16 * ks, pw);
            }
            const float2 s2 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
            const float sum = s2.x + s2.y;
            l = l * alpha + sum;
            if (j >= 1) {
                // O_t holds the products up to key tile j - 1 once that PV product has completed
                if (!(ok = mbar_wait(bar(AB_ODONE0 + t), (j - 1) & 1, MASK, abort_flag, prm.status, 139))) break;
                tc_fence_after();
                if (rescale) {
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        float o[32];
                        tmem_ld32(tl + co + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_st32f_nw(tl + co + c, o);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(AB_PREADY0 + t));
            if (quarter == 2) ATTN_PT(6 + t, j);
        }
        if (ok) ok = mbar_wait(bar(AB_ODONE0 + t), (nt - 1) & 1, MASK, abort_flag, prm.status, 140);
        uint8_t *qt = sm + Lo::kOffQ + t * Lo::kTile;
        if (ok) {
            // O_t / l as bf16 into Q_t's buffer (Q_t's last product has completed), as swizzled
            // [128][64] boxes
            tc_fence_after();
            const float inv = 1.f / l;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                float o[32];
                tmem_ld32(tl + co + c, o);
                uint8_t *box = qt + (c >> 6) * kABox;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint4 w;
                    w.x = pack_bf16(o[8 * qq + 0] * inv, o[8 * qq + 1] * inv);
                    w.y = pack_bf16(o[8 * qq + 2] * inv, o[8 * qq + 3] * inv);
                    w.z = pack_bf16(o[8 * qq + 4] * inv, o[8 * qq + 5] * inv);
                    w.w = pack_bf16(o[8 * qq + 6] * inv, o[8 * qq + 7] * inv);
                    *reinterpret_cast<uint4 *>(box + swz(r, ((c & 63) >> 3) + qq)) = w;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(AB_OSTAGED0 + t));
        }
        if (((warp - 2) & 3) == 0 && lane == 0 && ok) {
            if (mbar_wait(bar(AB_OSTAGED0 + t), 0, 1u, abort_flag, prm.status, 141)) {
                for (int x = 0; x < kBoxes; ++x)
                    tma_store_3d(&maps.o, smem_u32(qt) + x * kABox, hcol + 64 * x, q0 + kAQ * t, b);
                bulk_commit();
                bulk_wait0();
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// [batch][L][cols] view of a bf16 tensor whose tokens are ld elements apart: 3-D, so a tile
// that reaches past a sequence's end reads zeros and stores nothing there
bool make_map3(CUtensorMap *m, const void *base, int batch, int L, int cols, long long ld) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * (cuuint64_t)L};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_typed(const AttnArgs &a, cudaStream_t st) {
    using Lo = AttnLayout<D>;
    AttnMaps maps;
    memset(&maps, 0, sizeof maps);
    const int cols = a.H * D;
    if (!make_map3(&maps.q, a.q, a.batch, a.L, cols, a.ldq) || !make_map3(&maps.k, a.k, a.batch, a.L, cols, a.ldk) ||
        !make_map3(&maps.v, a.v, a.batch, a.L, cols, a.ldv) || !make_map3(&maps.o, a.o, a.batch, a.L, cols, a.ldo))
        return cudaErrorInvalidValue;
    AttnParams p{};
    p.L = a.L;
    p.ntiles = (a.L + kAKeys - 1) / kAKeys;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.status = a.status;
    p.wait_cycles = a.wait_cycles;
    cudaError_t e = cudaFuncSetAttribute(k_attention<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.L + kATiles * kAQ - 1) / (kATiles * kAQ)), (unsigned)a.H, (unsigned)a.batch);
    k_attention<D><<<grid, kAThreads, Lo::kSmem, st>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace

#ifdef SSD_TRACE
extern "C" int attn_debug_trace(unsigned long long *out, int n) {
    const int total = kATracePts * kATraceTiles;
    if (n < total) return -1;
    return cudaMemcpyFromSymbol(out, g_attn_trace, sizeof(unsigned long long) * total) == cudaSuccess ? total : -2;
}
#endif

bool attention_supported(int D) { return (D == 64 || D == 128) && get_encode() != nullptr; }

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st) {
    if (a.batch <= 0 || a.L <= 0 || a.H <= 0) return cudaSuccess;
    if (a.D == 64) return launch_typed<64>(a, st);
    if (a.D == 128) return launch_typed<128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace ssd
