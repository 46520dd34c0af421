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

// Persistent: one CTA per SM walks output tiles of 128 x 256 (tile t: rows 128 (t / nN), columns
// 256 (t % nN); CTAs that run together share an A row block, and W stays in L2).  Warp 0 feeds a
// 4-stage TMA ring (A box 128 x 64, W box 256 x 64, both K-major, 128-byte swizzle); warp 1 issues
// the MMAs (M 128, N 256, K 16) into one of two TMEM accumulators (256 columns each), so the
// epilogue warps 2-5 drain tile i while tile i + 1 accumulates.  The epilogue converts to bf16
// and stages each 128-column half of the tile in shared memory for a TMA store.
constexpr int kGM = 128, kGN = 256, kGK = 64;   // tile; K step of one 128-byte swizzled row
constexpr int kGStages = 4;
constexpr uint32_t kGATile = kGM * kGK * 2;     // 16 KB
constexpr uint32_t kGWTile = kGN * kGK * 2;     // 32 KB
constexpr uint32_t kGStage = kGATile + kGWTile;
constexpr uint32_t kGBox = 128 * 128;           // one [128 rows][64 bf16] output box, 16 KB
constexpr uint32_t kGOut = kGStages * kGStage;  // output staging: two boxes (half a tile)
constexpr uint32_t kGBar = kGOut + 2 * kGBox;
enum GemmBar {
    GB_FULL0 = 0,
    GB_EMPTY0 = GB_FULL0 + kGStages,
    GB_ACCFULL0 = GB_EMPTY0 + kGStages,         // two accumulators
    GB_ACCEMPTY0 = GB_ACCFULL0 + 2,
    GB_STAGED = GB_ACCEMPTY0 + 2,               // the four epilogue warps wrote the half tile
    GB_STAGEFREE,                               // the TMA store has read it
    GB_DONE,
    kGemmBars
};
constexpr uint32_t kGMisc = kGBar + kGemmBars * 8;
constexpr uint32_t kGemmSmem = kGMisc + 32 + 1024;
constexpr int kGemmThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
static_assert(kGemmSmem <= 232448, "shared memory budget");

struct GemmMaps {
    CUtensorMap a[2], w[2], d;                  // two (A, W) pairs summed over K; D the output
};
struct GemmParams {
    int M, N, k1, k2;                           // K of the first pair and of the second (0: none)
    int ntiles, ntn;                            // output tiles, tiles along N
    int *status;
    long long wait_cycles;
};

__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm_bf16(const __grid_constant__ GemmMaps maps,
                                                               const __grid_constant__ GemmParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto bar = [&](int i) { return sbase + kGBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kGMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kGMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk1 = prm.k1 / kGK, nk = nk1 + prm.k2 / kGK;
    const uint32_t MASK = 0xffffffffu;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *reinterpret_cast<volatile long long *>(abort_flag + 1) = prm.wait_cycles;
        for (int i = 0; i < kGemmBars; ++i)
            mbar_init(bar(i), (i == GB_ACCEMPTY0 || i == GB_ACCEMPTY0 + 1 || i == GB_STAGED) ? 4u : 1u);
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
            long long g = 0;                                  // k-steps issued so far, over all tiles
            bool ok = true;
            for (int t = blockIdx.x; t < prm.ntiles && ok; t += gridDim.x) {
                const int m0 = (t / prm.ntn) * kGM, n0 = (t % prm.ntn) * kGN;
                for (int kt = 0; kt < nk; ++kt, ++g) {
                    const int st = (int)(g % kGStages);
                    if (g >= kGStages &&
                        !(ok = mbar_wait(bar(GB_EMPTY0 + st), (uint32_t)((g / kGStages) - 1) & 1, 1u, abort_flag,
                                         prm.status, 121)))
                        break;
                    const int pr = kt < nk1 ? 0 : 1, kc = (kt < nk1 ? kt : kt - nk1) * kGK;
                    const uint32_t base = sbase + st * kGStage;
                    mbar_expect_tx(bar(GB_FULL0 + st), kGStage);
                    tma_load_2d(base, &maps.a[pr], kc, m0, bar(GB_FULL0 + st));
                    tma_load_2d(base + kGATile, &maps.w[pr], kc, n0, bar(GB_FULL0 + st));
                }
            }
            if (*abort_flag)
                for (long long q = g - 1; q >= 0 && q >= g - kGStages; --q)
                    mbar_drain(bar(GB_FULL0 + (int)(q % kGStages)), (uint32_t)(q / kGStages) & 1, prm.wait_cycles);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMAs (one elected lane)
        const uint32_t id = idesc(kGN, 0, 0);
        long long g = 0;
        int tc = 0;                                           // tiles of this CTA so far
        bool ok = true;
        for (int t = blockIdx.x; t < prm.ntiles && ok; t += gridDim.x, ++tc) {
            const int acc = tc & 1;
            // the accumulator is free once the epilogue has read tile tc - 2 out of it
            if (tc >= 2 &&
                !(ok = mbar_wait(bar(GB_ACCEMPTY0 + acc), ((tc >> 1) - 1) & 1, MASK, abort_flag, prm.status, 122)))
                break;
            tc_fence_after();
            for (int kt = 0; kt < nk; ++kt, ++g) {
                const int st = (int)(g % kGStages);
                if (!(ok = mbar_wait(bar(GB_FULL0 + st), (uint32_t)(g / kGStages) & 1, MASK, abort_flag, prm.status,
                                     123)))
                    break;
                tc_fence_after();
                const uint32_t base = sbase + st * kGStage;
                const SDesc da = make_sdesc(base, 16, 1024), dw = make_sdesc(base + kGATile, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < kGK / 16; ++ks)
                    mma_ss_w(tmem + 256u * acc, da.at(ks * 32), dw.at(ks * 32), id, (kt | ks) != 0);
                mma_commit_w(bar(GB_EMPTY0 + st));
            }
            if (!ok) break;
            mma_commit_w(bar(GB_ACCFULL0 + acc));
        }
        // every MMA issued has completed before TMEM is released
        mma_commit_w(bar(GB_DONE));
        if (lane == 0) mbar_drain(bar(GB_DONE), 0, prm.wait_cycles);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue: TMEM -> bf16 -> TMA store
        const int q = warp & 3, r = 32 * q + lane;
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const bool storer = warp == 2 && lane == 0;
        int tc = 0, h = 0;                                    // tiles, half tiles staged so far
        bool ok = true;
        for (int t = blockIdx.x; t < prm.ntiles && ok; t += gridDim.x, ++tc) {
            const int acc = tc & 1;
            const int m0 = (t / prm.ntn) * kGM, n0 = (t % prm.ntn) * kGN;
            if (!(ok = mbar_wait(bar(GB_ACCFULL0 + acc), (tc >> 1) & 1, MASK, abort_flag, prm.status, 124))) break;
            tc_fence_after();
            for (int half = 0; half < 2 && ok; ++half, ++h) {
                // the staging buffer is free once the previous half's store has read it
                if (h >= 1 && !(ok = mbar_wait(bar(GB_STAGEFREE), (h - 1) & 1, MASK, abort_flag, prm.status, 125)))
                    break;
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float v[32];
                    tmem_ld32(tl + 256u * acc + 128u * half + c0, v);
                    uint8_t *box = sm + kGOut + (c0 >> 6) * kGBox;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        uint4 o;
                        o.x = pack_bf16(v[8 * qq + 0], v[8 * qq + 1]);
                        o.y = pack_bf16(v[8 * qq + 2], v[8 * qq + 3]);
                        o.z = pack_bf16(v[8 * qq + 4], v[8 * qq + 5]);
                        o.w = pack_bf16(v[8 * qq + 6], v[8 * qq + 7]);
                        *reinterpret_cast<uint4 *>(box + swz(r, ((c0 & 63) >> 3) + qq)) = o;
                    }
                }
                if (half == 1) {
                    // the whole accumulator has been read: the MMA warp may reuse it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(GB_ACCEMPTY0 + acc));
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(GB_STAGED));
                if (storer) {
                    if ((ok = mbar_wait(bar(GB_STAGED), h & 1, 1u, abort_flag, prm.status, 126))) {
                        for (int x = 0; x < 2; ++x) {
                            const int nc = n0 + 128 * half + 64 * x;
                            if (nc < prm.N) tma_store_2d(&maps.d, sbase + kGOut + x * kGBox, nc, m0);
                        }
                        bulk_commit();
                        bulk_wait_read0();
                    }
                    mbar_arrive(bar(GB_STAGEFREE));
                }
                ok = __shfl_sync(MASK, ok ? 1 : 0, 0) != 0 && ok;
            }
        }
        if (storer) bulk_wait0();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// ------------------------------------------------------------------ conv + SiLU, dt softplus

// One thread: 4 consecutive channels of xBC (or 4 heads of dt) over a run of kConvT tokens of
// one sequence.  The thread first copies every input row it needs (8 bytes each) into its own
// column of shared memory with cp.async, so all of them are in flight at once and none holds a
// register; it reads back only what it copied itself, so no barrier is needed.  The taps and
// bias stay in registers and the inputs slide through a window.  Taps of the forward layer:
// token t + k - (K - 1); of the reverse layer: t - k + (K - 1) (the run is walked backwards);
// zero outside the sequence.  Four channels a thread (not eight) halve the staging a thread
// holds, so twice as many warps fit beside the same shared memory: the kernel is bound by
// latency, not by its arithmetic.
constexpr int kConvT = 32, kConvKMax = 8, kConvThreads = 128;

__device__ __forceinline__ float2 silu2(float2 v) {
    const float2 t = mul2(v, make_float2(-1.4426950408889634f, -1.4426950408889634f));
    float e0, e1, r0, r1;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(t.x));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(t.y));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(1.f + e0));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(1.f + e1));
    return mul2(v, make_float2(r0, r1));
}

__device__ __forceinline__ void conv_out(const MixerConvArgs &a, long long tok, int c0, const float2 (&acc)[2]) {
    uint32_t o[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const float2 s_ = silu2(acc[p]);
        o[p] = pack_bf16(s_.x, s_.y);
    }
    __nv_bfloat16 *dst;
    if (c0 < a.d_inner) dst = a.x + tok * a.d_inner + c0;
    else if (c0 < a.d_inner + a.N) dst = a.B + tok * a.N + (c0 - a.d_inner);
    else dst = a.C + tok * a.N + (c0 - a.d_inner - a.N);
    *reinterpret_cast<uint2 *>(dst) = make_uint2(o[0], o[1]);
}

__device__ __forceinline__ void unpack2x2(const uint2 &v, float2 (&f)[2]) {
    f[0] = unpack2(v.x);
    f[1] = unpack2(v.y);
}
__device__ __forceinline__ void unpack4x2(const uint4 &v, float2 (&f)[4]) {
    f[0] = unpack2(v.x); f[1] = unpack2(v.y); f[2] = unpack2(v.z); f[3] = unpack2(v.w);
}

// KT > 0: the conv width, fixed at compile time; KT = 0: the width a.K (at most kConvKMax)
template <int KT>
__global__ void __launch_bounds__(kConvThreads) k_conv_silu_dt(MixerConvArgs a) {
    constexpr int KM = KT > 0 ? KT : kConvKMax;
    extern __shared__ uint2 conv_stage[];   // [kConvT + KM - 1][kConvThreads]
    const int K = KT > 0 ? KT : a.K;
    const int groups_xbc = a.conv_dim / 4, groups = groups_xbc + a.H / 4;
    const int gidx = blockIdx.x * kConvThreads + threadIdx.x;
    if (gidx >= groups) return;
    const int runs = a.L / kConvT;
    const int b = blockIdx.y / runs, t0 = (blockIdx.y % runs) * kConvT;
    const long long seq0 = (long long)b * a.L;
    const bool is_dt = gidx >= groups_xbc;
    const int c0 = is_dt ? 4 * (gidx - groups_xbc) : 4 * gidx;          // channel (or head) of xBC (or dt)
    const int col = is_dt ? a.d_inner + a.conv_dim + c0 : a.d_inner + c0;  // its column in zxbcdt
    const int halo = is_dt ? 0 : K - 1;
    const int step = (is_dt || a.dir > 0) ? 1 : -1;
    const int first = step > 0 ? t0 : t0 + kConvT - 1;
    // row r of the column: the input at token first + step * (r - halo), zero outside the sequence
    // Two copy groups: the halo and the first half of the run, then the second half, so the
    // first half is computed while the second is still in flight.
    uint2 *mine = conv_stage + threadIdx.x;
    auto copy_rows = [&](int r0, int r1) {
        for (int r = r0; r < r1; ++r) {
            const int t = first + step * (r - halo);
            uint2 *dst = mine + r * kConvThreads;
            if (t < 0 || t >= a.L) {
                *dst = make_uint2(0u, 0u);
            } else {
                const __nv_bfloat16 *src = a.zxbcdt + (seq0 + t) * a.d_in_proj + col;
                asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    copy_rows(0, halo + kConvT / 2);
    copy_rows(halo + kConvT / 2, halo + kConvT);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    if (is_dt) {
        float bias[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) bias[e] = a.dt_bias[c0 + e];
#pragma unroll 4
        for (int i = 0; i < kConvT; ++i) {
            if (i == kConvT / 2) asm volatile("cp.async.wait_group 0;" ::: "memory");
            float2 v[2];
            unpack2x2(mine[i * kConvThreads], v);
            uint32_t o[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float r0 = v[e].x + bias[2 * e], r1 = v[e].y + bias[2 * e + 1];
                // softplus, with the linear branch above 20 (exp would dominate 1 there)
                const float s0 = r0 > 20.f ? r0 : log1pf(__expf(r0));
                const float s1 = r1 > 20.f ? r1 : log1pf(__expf(r1));
                o[e] = pack_bf16(s0, s1);
            }
            *reinterpret_cast<uint2 *>(a.dt + (seq0 + t0 + i) * a.H + c0) = make_uint2(o[0], o[1]);
        }
        return;
    }
    // wr[p][j]: the taps of channels (2p, 2p + 1) that multiply the input j steps back
    // (tap K - 1 - j), 0 past the width
    float2 wr[2][KM], bias[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        bias[p] = make_float2(a.conv_b[c0 + 2 * p], a.conv_b[c0 + 2 * p + 1]);
#pragma unroll
        for (int j = 0; j < KM; ++j)
            wr[p][j] = j < K ? make_float2(a.conv_w[(c0 + 2 * p) * K + (K - 1 - j)],
                                           a.conv_w[(c0 + 2 * p + 1) * K + (K - 1 - j)])
                             : make_float2(0.f, 0.f);
    }
    // win[j]: the input j steps back in the layer's order.  Before the first token's shift it
    // holds the token j + 1 steps back (rows halo - 1 down to 0, then zeros).
    float2 win[KM][2];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (j < halo) unpack2x2(mine[(halo - 1 - j) * kConvThreads], win[j]);
        else {
#pragma unroll
            for (int p = 0; p < 2; ++p) win[j][p] = make_float2(0.f, 0.f);
        }
    }
    // unrolled by 4 only: a fully unrolled run does not fit the instruction cache
#pragma unroll 4
    for (int i = 0; i < kConvT; ++i) {
        if (i == kConvT / 2) asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
        for (int j = KM - 1; j > 0; --j)
#pragma unroll
            for (int p = 0; p < 2; ++p) win[j][p] = win[j - 1][p];
        unpack2x2(mine[(halo + i) * kConvThreads], win[0]);
        float2 acc[2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float2 s_ = bias[p];
#pragma unroll
            for (int j = 0; j < KM; ++j) s_ = fma2(wr[p][j], win[j][p], s_);
            acc[p] = s_;
        }
        conv_out(a, seq0 + first + step * i, c0, acc);
    }
}

// ------------------------------------------------------------------ gated RMS norm

// One CTA per token, d_inner / (8 U) threads, each with U chunks of 8 channels (U loads of y
// and of z in flight): g = y * silu(z), computed once and kept in registers, then
// g / sqrt(mean(g^2) + eps) * w.  norm_w is read as float4 (16-byte aligned).
template <int U>
__global__ void __launch_bounds__(1024) k_gated_norm(MixerNormArgs a) {
    __shared__ float part[32];
    const long long tok = blockIdx.x;
    const int stride = 8 * blockDim.x;
    const __nv_bfloat16 *yrow = a.y + tok * a.d_inner, *zrow = a.zxbcdt + tok * a.d_in_proj;
    uint4 yv[U], zv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        yv[u] = *reinterpret_cast<const uint4 *>(yrow + 8 * threadIdx.x + u * stride);
        zv[u] = *reinterpret_cast<const uint4 *>(zrow + 8 * threadIdx.x + u * stride);
    }
    float2 g[U][4], ss2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float2 yf[4], zf[4];
        unpack4x2(yv[u], yf);
        unpack4x2(zv[u], zf);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            g[u][p] = mul2(yf[p], silu2(zf[p]));
            ss2 = fma2(g[u][p], g[u][p], ss2);
        }
    }
    float ss = ss2.x + ss2.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
    const float inv = rsqrtf(tot / a.d_inner + a.eps);
    const float2 inv2 = make_float2(inv, inv);
    __nv_bfloat16 *orow = a.out + tok * a.d_inner;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c0 = 8 * threadIdx.x + u * stride;
        const float4 w0 = *reinterpret_cast<const float4 *>(a.w + c0);
        const float4 w1 = *reinterpret_cast<const float4 *>(a.w + c0 + 4);
        const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                              make_float2(w1.z, w1.w)};
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 v = mul2(mul2(g[u][p], inv2), wp[p]);
            o[p] = pack_bf16(v.x, v.y);
        }
        *reinterpret_cast<uint4 *>(orow + c0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
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
            !make_map(&maps.w[p], p ? g.W2 : g.W1, g.N, K, 64, true, kGN))
            return cudaErrorInvalidValue;
    }
    if (!make_map(&maps.d, g.D, g.M, g.N, 64, true)) return cudaErrorInvalidValue;
    GemmParams p{};
    p.M = g.M; p.N = g.N; p.k1 = g.k1; p.k2 = g.k2;
    p.ntn = (g.N + kGN - 1) / kGN;
    p.ntiles = (g.M / kGM) * p.ntn;
    p.status = g.status; p.wait_cycles = g.wait_cycles;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int grid = p.ntiles < sms ? p.ntiles : sms;
    k_gemm_bf16<<<grid, kGemmThreads, kGemmSmem, st>>>(maps, p);
    return cudaGetLastError();
}

cudaError_t launch_conv_silu_dt(const MixerConvArgs &a, cudaStream_t st) {
    if (a.L % kConvT != 0 || a.K < 1 || a.K > kConvKMax) return cudaErrorInvalidValue;
    const int groups = a.conv_dim / 4 + a.H / 4;
    dim3 grid((groups + kConvThreads - 1) / kConvThreads, (unsigned)((long long)a.batch * (a.L / kConvT)));
    auto run = [&](auto kernel, int km) -> cudaError_t {
        const int smem = (kConvT + km - 1) * kConvThreads * (int)sizeof(uint2);
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kernel<<<grid, kConvThreads, smem, st>>>(a);
        return cudaGetLastError();
    };
    switch (a.K) {
        case 2: return run(k_conv_silu_dt<2>, 2);
        case 3: return run(k_conv_silu_dt<3>, 3);
        case 4: return run(k_conv_silu_dt<4>, 4);
        default: return run(k_conv_silu_dt<0>, kConvKMax);
    }
}

cudaError_t launch_gated_norm(const MixerNormArgs &a, cudaStream_t st) {
    if (a.d_inner % 512 != 0 || a.d_inner > 16384 || (reinterpret_cast<uintptr_t>(a.w) & 15) != 0)
        return cudaErrorInvalidValue;
    const unsigned tokens = (unsigned)((long long)a.batch * a.L);
    if (a.d_inner % 1024 == 0 && a.d_inner <= 8192)
        k_gated_norm<4><<<tokens, a.d_inner / 32, 0, st>>>(a);
    else
        k_gated_norm<2><<<tokens, a.d_inner / 16, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ssd
