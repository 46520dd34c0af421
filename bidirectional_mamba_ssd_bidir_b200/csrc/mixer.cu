// mixer.cu -- the Mamba-2 block around the scan: the two projections (tcgen05
// GEMMs), the depthwise convolution with SiLU and the dt softplus, and the
// gated RMS norm.
//
// The DiffuMamba page ("DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", technical summary, section 2) builds its mixer from two
// independent bidirectional Mamba-2 layers; the inside of a layer is read as
// the standard Mamba-2 block:
//
//   zxbcdt = u W_in^T;  xBC = silu(conv(xBC) + b);  dt = softplus(dt + dt_bias);
//   y = scan(x, dt, A, B, C, D);  yn = rmsnorm(y * silu(z)) * w;  out = yn W_out^T
//
// and the mixer is layer_f(u) + flip(layer_r(flip(u))).  The reverse layer is
// run in place, without flipping anything: its projections act per token, its
// convolution looks at the later tokens, and its scan runs in reverse.  The
// output projection of both layers is one product over the concatenated
// inner dimension: [yn_f | yn_r] [W_out_f | W_out_r]^T.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "mixer.cuh"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace {

// ------------------------------------------------------------------ GEMM: D[M][N] = A[M][K] W[N][K]^T

constexpr int kGM = 128, kGN = 128, kGK = 64;   // tile; K step of one 128-byte swizzled row
constexpr int kGStages = 3;
constexpr uint32_t kGTile = kGM * kGK * 2;      // 16 KB (A tile and W tile alike)
constexpr uint32_t kGStage = 2 * kGTile;
constexpr uint32_t kGBar = kGStages * kGStage;
enum GemmBar { GB_FULL0 = 0, GB_EMPTY0 = GB_FULL0 + kGStages, GB_DONE = GB_EMPTY0 + kGStages, kGemmBars };
constexpr uint32_t kGMisc = kGBar + kGemmBars * 8;
constexpr uint32_t kGemmSmem = kGMisc + 32 + 1024;
constexpr int kGemmThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

struct GemmMaps {
    CUtensorMap a[2], w[2], d;                  // two (A, W) pairs summed over K; D the output
};
struct GemmParams {
    int M, N, k1, k2;                           // K of the first pair and of the second (0: none)
    int *status;
    long long wait_cycles;
};

__global__ void __launch_bounds__(kGemmThreads, 2) k_gemm_bf16(const __grid_constant__ GemmMaps maps,
                                                               const __grid_constant__ GemmParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kGBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kGMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kGMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kGN, m0 = blockIdx.y * kGM;
    const int nk1 = prm.k1 / kGK, nk = nk1 + prm.k2 / kGK;
    const uint32_t MASK = 0xffffffffu;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kGemmBars; ++i) mbar_init(bar(i), 1);
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

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < nk; ++kt) {
                const int st = kt % kGStages;
                if (kt >= kGStages &&
                    !mbar_wait(bar(GB_EMPTY0 + st), ((kt / kGStages) - 1) & 1, 1u, abort_flag, prm.status, 121))
                    break;
                const int pr = kt < nk1 ? 0 : 1, kc = (kt < nk1 ? kt : kt - nk1) * kGK;
                const uint32_t base = sbase + st * kGStage;
                mbar_expect_tx(bar(GB_FULL0 + st), kGStage);
                tma_load_2d(base, &maps.a[pr], kc, m0, bar(GB_FULL0 + st));
                tma_load_2d(base + kGTile, &maps.w[pr], kc, n0, bar(GB_FULL0 + st));
                issued = kt + 1;
            }
            if (*abort_flag)
                for (int kt = issued - 1; kt >= 0 && kt >= issued - kGStages; --kt)
                    mbar_drain(bar(GB_FULL0 + kt % kGStages), (kt / kGStages) & 1, prm.wait_cycles);
        }
        __syncwarp();
    } else if (warp == 1) {
        const uint32_t id = idesc(kGN, 0, 0);
        bool ok = true;
        for (int kt = 0; kt < nk && ok; ++kt) {
            const int st = kt % kGStages;
            if (!(ok = mbar_wait(bar(GB_FULL0 + st), (kt / kGStages) & 1, MASK, abort_flag, prm.status, 122))) break;
            tc_fence_after();
            const uint32_t base = sbase + st * kGStage;
            const SDesc da = make_sdesc(base, kGTile, 1024), dw = make_sdesc(base + kGTile, kGTile, 1024);
#pragma unroll
            for (int ks = 0; ks < kGK / 16; ++ks) mma_ss_w(tmem, da.at(ks * 32), dw.at(ks * 32), id, (kt | ks) != 0);
            mma_commit_w(bar(GB_EMPTY0 + st));
        }
        mma_commit_w(bar(GB_DONE));
        if (lane == 0 && !ok) mbar_drain(bar(GB_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // epilogue: TMEM lane quarter warp % 4 (rows), all 128 columns; bf16 into two swizzled
        // [128][64] halves (the pipeline stages are free once every MMA has completed), then TMA
        if (mbar_wait(bar(GB_DONE), 0, MASK, abort_flag, prm.status, 123)) {
            tc_fence_after();
            const int q = warp & 3, r = 32 * q + lane;
            const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < kGN; c0 += 32) {
                float v[32];
                tmem_ld32(tl + c0, v);
                uint8_t *half = sm + (c0 >> 6) * kGTile;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    uint4 o;
                    o.x = pack_bf16(v[8 * qq + 0], v[8 * qq + 1]);
                    o.y = pack_bf16(v[8 * qq + 2], v[8 * qq + 3]);
                    o.z = pack_bf16(v[8 * qq + 4], v[8 * qq + 5]);
                    o.w = pack_bf16(v[8 * qq + 6], v[8 * qq + 7]);
                    *reinterpret_cast<uint4 *>(half + swz(r, ((c0 & 63) >> 3) + qq)) = o;
                }
            }
            fence_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 64 && !*abort_flag) {
        for (int hf = 0; hf < 2; ++hf)
            if (n0 + 64 * hf < prm.N) tma_store_2d(&maps.d, sbase + hf * kGTile, n0 + 64 * hf, m0);
        bulk_commit();
        bulk_wait0();
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
    }
}

// ------------------------------------------------------------------ conv + SiLU, dt softplus

// One thread: 8 consecutive channels of xBC (or 8 heads of dt) of one token.  Taps of the
// forward layer: token t + k - (K - 1); of the reverse layer: t - k + (K - 1); zero outside the
// sequence.
__global__ void __launch_bounds__(256) k_conv_silu_dt(MixerConvArgs a) {
    const int groups_xbc = a.conv_dim / 8, groups_dt = a.H / 8, groups = groups_xbc + groups_dt;
    const long long total = (long long)a.batch * a.L * groups;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int gidx = (int)(i % groups);
        const long long tok = i / groups;                 // b * L + t
        const int t = (int)(tok % a.L);
        const __nv_bfloat16 *row = a.zxbcdt + tok * a.d_in_proj;
        if (gidx < groups_xbc) {
            const int c0 = 8 * gidx;
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = a.conv_b[c0 + e];
            for (int k = 0; k < a.K; ++k) {
                const int tt = a.dir > 0 ? t + k - (a.K - 1) : t - k + (a.K - 1);
                if (tt < 0 || tt >= a.L) continue;
                const uint4 v = *reinterpret_cast<const uint4 *>(row + (long long)(tt - t) * a.d_in_proj + a.d_inner + c0);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[2 * e] = fmaf(a.conv_w[(c0 + 2 * e) * a.K + k], bf16lo(w4[e]), acc[2 * e]);
                    acc[2 * e + 1] = fmaf(a.conv_w[(c0 + 2 * e + 1) * a.K + k], bf16hi(w4[e]), acc[2 * e + 1]);
                }
            }
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float s0 = acc[2 * e] / (1.f + __expf(-acc[2 * e]));
                const float s1 = acc[2 * e + 1] / (1.f + __expf(-acc[2 * e + 1]));
                o[e] = pack_bf16(s0, s1);
            }
            __nv_bfloat16 *dst;
            if (c0 < a.d_inner) dst = a.x + tok * a.d_inner + c0;
            else if (c0 < a.d_inner + a.N) dst = a.B + tok * a.N + (c0 - a.d_inner);
            else dst = a.C + tok * a.N + (c0 - a.d_inner - a.N);
            *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
        } else {
            const int h0 = 8 * (gidx - groups_xbc);
            const uint4 v = *reinterpret_cast<const uint4 *>(row + a.d_inner + a.conv_dim + h0);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float r0 = bf16lo(w4[e]) + a.dt_bias[h0 + 2 * e], r1 = bf16hi(w4[e]) + a.dt_bias[h0 + 2 * e + 1];
                // softplus, with the linear branch above 20 (exp would dominate 1 there)
                const float s0 = r0 > 20.f ? r0 : log1pf(__expf(r0));
                const float s1 = r1 > 20.f ? r1 : log1pf(__expf(r1));
                o[e] = pack_bf16(s0, s1);
            }
            *reinterpret_cast<uint4 *>(a.dt + tok * a.H + h0) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// ------------------------------------------------------------------ gated RMS norm

// One CTA per token, one thread per 8 channels (d_inner / 8 threads, whole warps):
// g = y * silu(z) over d_inner, g / sqrt(mean(g^2) + eps) * w.
__global__ void __launch_bounds__(1024) k_gated_norm(MixerNormArgs a) {
    __shared__ float part[32];
    const long long tok = blockIdx.x;
    const int c0 = threadIdx.x * 8;
    const uint4 yv = *reinterpret_cast<const uint4 *>(a.y + tok * a.d_inner + c0);
    const uint4 zv = *reinterpret_cast<const uint4 *>(a.zxbcdt + tok * a.d_in_proj + c0);
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w}, zw[4] = {zv.x, zv.y, zv.z, zv.w};
    float g[8];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float z0 = bf16lo(zw[e]), z1 = bf16hi(zw[e]);
        g[2 * e] = bf16lo(yw[e]) * (z0 / (1.f + __expf(-z0)));
        g[2 * e + 1] = bf16hi(yw[e]) * (z1 / (1.f + __expf(-z1)));
        ss = fmaf(g[2 * e], g[2 * e], fmaf(g[2 * e + 1], g[2 * e + 1], ss));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const int nw = blockDim.x >> 5;
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < nw; ++w) tot += part[w];
    const float inv = rsqrtf(tot / a.d_inner + a.eps);
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = pack_bf16(g[2 * e] * inv * a.w[c0 + 2 * e], g[2 * e + 1] * inv * a.w[c0 + 2 * e + 1]);
    *reinterpret_cast<uint4 *>(a.out + tok * a.d_inner + c0) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

bool mixer_gemm_supported(int M, int N, int K) {
    return M > 0 && N > 0 && K > 0 && M % kGM == 0 && K % kGK == 0 && N % 8 == 0 && get_encode() != nullptr;
}

cudaError_t launch_gemm_bf16(const GemmArgs &g, cudaStream_t st) {
    GemmMaps maps;
    memset(&maps, 0, sizeof maps);
    // A: [M][K] (box 64 x 128), W: [N][K] (box 64 x 128), D: [M][N] (box 64 x 128), all swizzled
    for (int p = 0; p < (g.k2 ? 2 : 1); ++p) {
        const int K = p ? g.k2 : g.k1;
        if (!make_map(&maps.a[p], p ? g.A2 : g.A1, g.M, K, 64, true) ||
            !make_map(&maps.w[p], p ? g.W2 : g.W1, g.N, K, 64, true))
            return cudaErrorInvalidValue;
    }
    if (!make_map(&maps.d, g.D, g.M, g.N, 64, true)) return cudaErrorInvalidValue;
    GemmParams p{};
    p.M = g.M; p.N = g.N; p.k1 = g.k1; p.k2 = g.k2;
    p.status = g.status; p.wait_cycles = g.wait_cycles;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((g.N + kGN - 1) / kGN, g.M / kGM);
    k_gemm_bf16<<<grid, kGemmThreads, kGemmSmem, st>>>(maps, p);
    return cudaGetLastError();
}

cudaError_t launch_conv_silu_dt(const MixerConvArgs &a, cudaStream_t st) {
    const long long total = (long long)a.batch * a.L * (a.conv_dim / 8 + a.H / 8);
    const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
    k_conv_silu_dt<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gated_norm(const MixerNormArgs &a, cudaStream_t st) {
    if (a.d_inner % 256 != 0 || a.d_inner > 8192) return cudaErrorInvalidValue;
    k_gated_norm<<<(unsigned)((long long)a.batch * a.L), a.d_inner / 8, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ssd
