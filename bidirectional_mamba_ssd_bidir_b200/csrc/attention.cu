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
// One CTA per (128 queries, head, sequence), walking the keys in tiles of 128:
//
//   S_j  = Q K_j^T                 SS MMA into TMEM (two buffers, so the product for tile
//                                  j + 1 runs while tile j is in the softmax)
//   P_j  = 2^(S_j c - m)           CUDA cores, one thread per query row; bf16, written over
//                                  its own S buffer in TMEM (c = scale log2 e)
//   O   += P_j V_j                 TS MMA: A = P from TMEM, B = V (MN-major) from shared memory
//
// The reference m of a row follows the row maximum lazily: it moves only when a tile's maximum
// exceeds it by more than 8 (log2 units), so p <= 2^8 and O (in TMEM) is rescaled by 2^(m_old
// - m_new) only on those tiles.  The row sum l accumulates the bf16-rounded p the product
// uses; the epilogue writes O / l.  Tiles reach past the sequence's end as zeros (3-D tensor
// maps clip at each sequence); those keys are masked to p = 0 and those query rows are not
// stored.
//
// Warps (192 threads): warp 0 issues the TMA loads, warp 1 owns TMEM and issues the MMAs, warps
// 2-5 run the softmax (TMEM lane quarter warp % 4) and the epilogue.  Every wait is bounded;
// a wait that runs out records its code in the status word and the CTA winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "attention.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

constexpr int kAQ = 128;                       // query rows per CTA (= TMEM lanes)
constexpr int kAKeys = 128;                    // keys per tile
constexpr int kAThreads = 192;
constexpr int kAStages = 2;                    // K/V tiles in flight
constexpr uint32_t kABox = 128 * 128;          // one [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kColO = 256;                // TMEM: S/P buffers at 0 and 128, O at 256

enum AttnBar {
    AB_QFULL = 0,
    AB_KFULL0,
    AB_VFULL0 = AB_KFULL0 + kAStages,
    AB_KVEMPTY0 = AB_VFULL0 + kAStages,
    AB_SFULL0 = AB_KVEMPTY0 + kAStages,
    AB_PREADY0 = AB_SFULL0 + 2,
    AB_ODONE = AB_PREADY0 + 2,
    AB_OSTAGED,
    AB_DONE,
    kAttnBars
};

template <int D>
struct AttnLayout {
    static constexpr uint32_t kTile = (D / 64) * kABox;          // a [128][D] tile
    static constexpr uint32_t kOffQ = 0;                         // Q; the output tile at the end
    static constexpr uint32_t kOffKV = kTile;                    // stage s: K at + 2 s kTile, V after it
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
    const int q0 = blockIdx.x * kAQ, hcol = blockIdx.y * D, b = blockIdx.z;
    const int nt = prm.ntiles;
    const uint32_t MASK = 0xffffffffu;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kAttnBars; ++i)
            mbar_init(bar(i), (i == AB_PREADY0 || i == AB_PREADY0 + 1 || i == AB_OSTAGED) ? 4u : 1u);
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
            mbar_expect_tx(bar(AB_QFULL), Lo::kTile);
            for (int x = 0; x < kBoxes; ++x)
                tma_load_3d(sbase + Lo::kOffQ + x * kABox, &maps.q, hcol + 64 * x, q0, b, bar(AB_QFULL));
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int s = j % kAStages;
                // the stage is free once the PV product of tile j - kAStages has completed
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
        const uint32_t id_s = idesc(128, 0, 0);    // S = Q K^T: M = queries, N = keys, K = d
        const uint32_t id_o = idesc(D, 0, 1);      // O += P V: M = queries, N = d, K = keys
        // Q and K K-major (rows of 128 bytes, 8-row groups 1 KB apart, 64-column boxes kABox
        // apart); V MN-major (64-column chunks kABox apart, 8-key groups 1 KB apart)
        const SDesc dq = make_sdesc(sbase + Lo::kOffQ, 16, 1024);
        bool ok = mbar_wait(bar(AB_QFULL), 0, MASK, abort_flag, prm.status, 132);
        auto issue_s = [&](int j) -> bool {
            const int s = j % kAStages;
            if (!mbar_wait(bar(AB_KFULL0 + s), (j / kAStages) & 1, MASK, abort_flag, prm.status, 133)) return false;
            // S buffer j & 1 holds P of tile j - 2 until that tile's PV product has completed
            if (j >= 2 && !mbar_wait(bar(AB_ODONE), (j - 2) & 1, MASK, abort_flag, prm.status, 134)) return false;
            tc_fence_after();
            const SDesc dk = make_sdesc(sbase + Lo::kOffKV + s * 2 * Lo::kTile, 16, 1024);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (ks >> 2) * kABox + (ks & 3) * 32;
                mma_ss_w(tmem + 128u * (j & 1), dq.at(off), dk.at(off), id_s, ks > 0);
            }
            mma_commit_w(bar(AB_SFULL0 + (j & 1)));
            return true;
        };
        if (ok) ok = issue_s(0);
        for (int j = 0; j < nt && ok; ++j) {
            if (j + 1 < nt && !(ok = issue_s(j + 1))) break;
            const int s = j % kAStages;
            if (!(ok = mbar_wait(bar(AB_PREADY0 + (j & 1)), (j >> 1) & 1, MASK, abort_flag, prm.status, 135))) break;
            if (!(ok = mbar_wait(bar(AB_VFULL0 + s), (j / kAStages) & 1, MASK, abort_flag, prm.status, 136))) break;
            tc_fence_after();
            const SDesc dv = make_sdesc(sbase + Lo::kOffKV + s * 2 * Lo::kTile + Lo::kTile, kABox, 1024);
            // A = P (keys 16 ks .. 16 ks + 15 at TMEM columns [16 ks, 16 ks + 8) of the buffer)
#pragma unroll
            for (int ks = 0; ks < kAKeys / 16; ++ks)
                mma_ts_w(tmem + kColO, tmem + 128u * (j & 1) + 16 * ks, dv.at(ks * 2048), id_o, (j | ks) != 0);
            mma_commit_w(bar(AB_ODONE));
            mma_commit_w(bar(AB_KVEMPTY0 + s));
        }
        // every MMA issued has completed before TMEM is released
        mma_commit_w(bar(AB_DONE));
        if (lane == 0) mbar_drain(bar(AB_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax, epilogue
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;                       // query row = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
        float m_ref = 0.f, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const uint32_t sb = 128u * (j & 1);
            if (!(ok = mbar_wait(bar(AB_SFULL0 + (j & 1)), (j >> 1) & 1, MASK, abort_flag, prm.status, 137))) break;
            tc_fence_after();
            float t[128];
            tmem_ld32x2(tl + sb, tl + sb + 32, t, t + 32);
            tmem_ld32x2(tl + sb + 64, tl + sb + 96, t + 64, t + 96);
            const int valid = prm.L - j * kAKeys;               // keys of this tile inside the sequence
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                t[i] = i < valid ? t[i] * prm.scale_log2 : -INFINITY;
                mx = fmaxf(mx, t[i]);
            }
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
            // P = 2^(t - m_ref) as bf16 over the S buffer; l sums the rounded values
            float sum = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t pw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    pw[i] = pack_bf16(ex2_ftz(t[16 * ks + 2 * i] - m_ref), ex2_ftz(t[16 * ks + 2 * i + 1] - m_ref));
                    sum += bf16lo(pw[i]) + bf16hi(pw[i]);
                }
                tmem_st8_nw(tl + sb + 16 * ks, pw);
            }
            l = l * alpha + sum;
            if (j >= 1) {
                // O holds the products up to tile j - 1 once that PV product has completed
                if (!(ok = mbar_wait(bar(AB_ODONE), (j - 1) & 1, MASK, abort_flag, prm.status, 138))) break;
                tc_fence_after();
                if (rescale) {
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        float o[32];
                        tmem_ld32(tl + kColO + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_st32f_nw(tl + kColO + c, o);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(AB_PREADY0 + (j & 1)));
        }
        if (ok) ok = mbar_wait(bar(AB_ODONE), (nt - 1) & 1, MASK, abort_flag, prm.status, 139);
        if (ok) {
            // O / l as bf16 into the Q buffer (every MMA has completed), as swizzled [128][64] boxes
            tc_fence_after();
            const float inv = 1.f / l;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                float o[32];
                tmem_ld32(tl + kColO + c, o);
                uint8_t *box = sm + Lo::kOffQ + (c >> 6) * kABox;
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
            if (lane == 0) mbar_arrive(bar(AB_OSTAGED));
        }
        if (warp == 2 && lane == 0 && ok) {
            if (mbar_wait(bar(AB_OSTAGED), 0, 1u, abort_flag, prm.status, 140)) {
                for (int x = 0; x < kBoxes; ++x)
                    tma_store_3d(&maps.o, sbase + Lo::kOffQ + x * kABox, hcol + 64 * x, q0, b);
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
    dim3 grid((unsigned)((a.L + kAQ - 1) / kAQ), (unsigned)a.H, (unsigned)a.batch);
    k_attention<D><<<grid, kAThreads, Lo::kSmem, st>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace

bool attention_supported(int D) { return (D == 64 || D == 128) && get_encode() != nullptr; }

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st) {
    if (a.batch <= 0 || a.L <= 0 || a.H <= 0) return cudaSuccess;
    if (a.D == 64) return launch_typed<64>(a, st);
    if (a.D == 128) return launch_typed<128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace ssd
