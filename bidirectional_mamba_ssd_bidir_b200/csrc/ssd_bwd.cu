// ssd_bwd.cu -- gradients of one direction of the SSD scan, on the CUDA cores
// (float32 throughout).
//
// Training the layers that run the scan needs its reverse-mode derivative (the
// DiffuMamba page, technical summary, section 2, trains the Mamba backbone
// with the masked-diffusion objective).  With k the scan position, cs_k the
// cumulative A dt in scan order, the state S_k = a_k S_{k-1} + dt_k x_k B_k^T
// (a_k = exp(dt_k A)) and y_k = S_k C_k + D x_k, the derivative of L with
// respect to S_k is
//     G_k = gy_k C_k^T + a_{k+1} G_{k+1}
// and
//     dx_k  = dt_k G_k B_k + D gy_k
//     dB_k  = dt_k G_k^T x_k                 (summed over the heads of a group)
//     dC_k  = S_k^T gy_k                     (summed over the heads of a group)
//     ddt_k = u_k + A sum_{k' >= k} gcs_k',   u_k = <G_k, x_k B_k^T>
//     dA    = sum_k dt_k sum_{k' >= k} gcs_k'
//     dD    = sum_k <gy_k, x_k>
// where gcs_k = <gy_k, y_k - D x_k> - dt_k u_k is the derivative with respect
// to cs_k (the decays exp(cs_t - cs_s) differentiate into +gcs at the output
// position and -gcs at the input position).
//
// Chunked evaluation (Q positions per chunk, as in the forward pass):
//   1. per chunk, in parallel: the chunk's own state sum and the adjoint's own
//      sum  Z_c = sum_k exp(cs_k) gy_k C_k^T  (cs from the chunk start),
//   2. per (batch, head): the forward pass over chunks (state entering each
//      chunk) and the reverse pass (adjoint entering each chunk from the
//      right: Gin_{c-1} = Z_c + exp(cs_last) Gin_c),
//   3. per chunk, in parallel: every per-position gradient from the chunk's
//      Q x Q pair terms and the two entering states,
//   4. per (batch, head): the suffix sums of gcs that give ddt and dA,
//   5. the sums over the heads of a group (dB, dC) and over the batch (dA, dD).
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kT = 256;       // threads per CTA
constexpr int kTC = 512;      // threads per CTA of the per-chunk gradient kernel (more warps hide its
                              // shared-memory latency; one CTA per SM fits its shared memory)

// Offset of the P x N chunk state (or adjoint) of (b, h, chunk c) in a.sf / a.sg.  The heads of
// one chunk are neighbours, so the state passes, which walk all heads chunk by chunk, touch one
// contiguous range at a time instead of addresses a power of two apart.
__device__ __forceinline__ size_t chunk_slot(const BwdArgs &a, int b, int h, int c, int PN) {
    return (((size_t)b * a.nc + c) * a.H + h) * (size_t)PN;
}

// Eight consecutive values of a 16-byte aligned row, as float.
template <typename T> __device__ __forceinline__ void ld8(const T *p, float (&v)[8]);
template <> __device__ __forceinline__ void ld8<float>(const float *p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> __device__ __forceinline__ void ld8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Eight floats to two 16-byte aligned addresses HALF apart (HALF = 4: eight consecutive).
template <int HALF = 4>
__device__ __forceinline__ void st8(float *d, const float (&v)[8]) {
    *reinterpret_cast<float4 *>(d) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(d + HALF) = make_float4(v[4], v[5], v[6], v[7]);
}

// Rows 0 .. Q-1 of two [token][W] arrays that share their row addresses (x and gy, or B and C)
// for one chunk, eight values per unit.  Every unit of this thread is loaded before any is
// handed to op(k, w0, va, vb), so that the loads are in flight together.
template <typename T, int W, int NT, typename RowOff, typename Op>
__device__ __forceinline__ void load_rows2(int Q, const T *ga, const T *gb, RowOff rowoff, Op op) {
    constexpr int WU = W / 8, MAXU = (64 * WU + NT - 1) / NT;
    float va[MAXU][8], vb[MAXU][8];
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
        const int i = threadIdx.x + NT * u;
        if (i < Q * WU) {
            const size_t o = rowoff(i / WU) + 8 * (i % WU);
            ld8<T>(ga + o, va[u]);
            ld8<T>(gb + o, vb[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
        const int i = threadIdx.x + NT * u;
        if (i < Q * WU) op(i / WU, 8 * (i % WU), va[u], vb[u]);
    }
}

// Inclusive prefix sum of A*dt over one chunk in scan order (cs[]), and dt (dts[]).
template <typename T>
__device__ void bwd_cumsum(const BwdArgs &a, int b, int h, int c, float *cs, float *dts) {
    __shared__ float wt[kTC / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float v = 0.f;
    if (tid < a.Q) {
        const int t = tok(c * a.Q + tid, a.L, a.dir);
        v = ldf<T>((const T *)a.dt, ((size_t)b * a.L + t) * a.H + h);
        dts[tid] = v;
    }
    float s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += u;
    }
    if (lane == 31) wt[warp] = s;
    __syncthreads();
    float base = 0.f;
    for (int w = 0; w < warp; ++w) base += wt[w];
    if (tid < a.Q) cs[tid] = a.A[h] * (base + s);
    __syncthreads();
}

// Step 1: the chunk's own forward state sum  sum_k exp(cs_last - cs_k) dt_k x_k B_k^T  and the
// adjoint's own sum  sum_k exp(cs_k) gy_k C_k^T.
template <typename T, int P, int N>
__global__ void __launch_bounds__(kT) k_bwd_chunk_sums(BwdArgs a) {
    constexpr int E = P * N / kT;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int Q = a.Q, g = h / (a.H / a.G);
    extern __shared__ __align__(16) float sm[];
    float *cs = sm, *dts = cs + 64, *xw = dts + 64, *gw = xw + Q * P, *bs = gw + Q * P, *cc = bs + Q * N;
    auto xrow = [&](int k) { return (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.H + h) * P; };
    auto brow = [&](int k) { return (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.G + g) * N; };
    load_rows2<T, N, kT>(Q, (const T *)a.B, (const T *)a.C, brow,
                         [&](int k, int n, const float (&vb)[8], const float (&vc)[8]) {
                             st8(bs + k * N + n, vb);
                             st8(cc + k * N + n, vc);
                         });
    bwd_cumsum<T>(a, b, h, c, cs, dts);
    const float cl = cs[Q - 1];
    load_rows2<T, P, kT>(Q, (const T *)a.x, (const T *)a.gy, xrow,
                         [&](int k, int p, const float (&vx)[8], const float (&vg)[8]) {
                             const float wx = expf(cl - cs[k]) * dts[k], wg = expf(cs[k]);
                             float ox[8], og[8];
#pragma unroll
                             for (int e = 0; e < 8; ++e) {
                                 ox[e] = wx * vx[e];
                                 og[e] = wg * vg[e];
                             }
                             st8(xw + k * P + p, ox);
                             st8(gw + k * P + p, og);
                         });
    __syncthreads();
    const size_t base = chunk_slot(a, b, h, c, P * N);
    if constexpr (E == 32 && N == 4 * 32 && P == 8 * (kT / 32)) {
        // 4 columns x 8 rows of each sum per thread: lane = column quad n0, warp = row octet p0.
        // B and C rows are read as whole-warp vectors, the row weights as broadcasts.
        const int n0 = 4 * (threadIdx.x & 31), p0 = 8 * (threadIdx.x >> 5);
        float sf[8][4], sg[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) sf[i][j] = sg[i][j] = 0.f;
#pragma unroll 2
        for (int k = 0; k < Q; ++k) {
            const float4 bv = *reinterpret_cast<const float4 *>(bs + k * N + n0);
            const float4 cv = *reinterpret_cast<const float4 *>(cc + k * N + n0);
            const float b4[4] = {bv.x, bv.y, bv.z, bv.w}, c4[4] = {cv.x, cv.y, cv.z, cv.w};
            float xv[8], gv[8];
            const float4 x0 = *reinterpret_cast<const float4 *>(xw + k * P + p0);
            const float4 x1 = *reinterpret_cast<const float4 *>(xw + k * P + p0 + 4);
            const float4 g0 = *reinterpret_cast<const float4 *>(gw + k * P + p0);
            const float4 g1 = *reinterpret_cast<const float4 *>(gw + k * P + p0 + 4);
            xv[0] = x0.x; xv[1] = x0.y; xv[2] = x0.z; xv[3] = x0.w; xv[4] = x1.x; xv[5] = x1.y; xv[6] = x1.z; xv[7] = x1.w;
            gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w; gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sf[i][j] = fmaf(xv[i], b4[j], sf[i][j]);
                    sg[i][j] = fmaf(gv[i], c4[j], sg[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            *reinterpret_cast<float4 *>(a.sf + base + (size_t)(p0 + i) * N + n0) =
                make_float4(sf[i][0], sf[i][1], sf[i][2], sf[i][3]);
            *reinterpret_cast<float4 *>(a.sg + base + (size_t)(p0 + i) * N + n0) =
                make_float4(sg[i][0], sg[i][1], sg[i][2], sg[i][3]);
        }
    } else {
        // thread: column n and E consecutive rows p0 .. p0 + E - 1, so that the row weights of one k
        // are read as whole vectors (the same for every lane of a warp when N >= 32)
        float sf[E], sg[E];
#pragma unroll
        for (int j = 0; j < E; ++j) sf[j] = sg[j] = 0.f;
        const int n = threadIdx.x % N, p0 = (threadIdx.x / N) * E;
#pragma unroll 2
        for (int k = 0; k < Q; ++k) {
            const float bv = bs[k * N + n], cv = cc[k * N + n];
            if constexpr (E % 4 == 0) {
#pragma unroll
                for (int j = 0; j < E; j += 4) {
                    const float4 xv = *reinterpret_cast<const float4 *>(xw + k * P + p0 + j);
                    const float4 gv = *reinterpret_cast<const float4 *>(gw + k * P + p0 + j);
                    sf[j] = fmaf(xv.x, bv, sf[j]); sf[j + 1] = fmaf(xv.y, bv, sf[j + 1]);
                    sf[j + 2] = fmaf(xv.z, bv, sf[j + 2]); sf[j + 3] = fmaf(xv.w, bv, sf[j + 3]);
                    sg[j] = fmaf(gv.x, cv, sg[j]); sg[j + 1] = fmaf(gv.y, cv, sg[j + 1]);
                    sg[j + 2] = fmaf(gv.z, cv, sg[j + 2]); sg[j + 3] = fmaf(gv.w, cv, sg[j + 3]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < E; ++j) {
                    sf[j] = fmaf(xw[k * P + p0 + j], bv, sf[j]);
                    sg[j] = fmaf(gw[k * P + p0 + j], cv, sg[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < E; ++j) {
            a.sf[base + (size_t)(p0 + j) * N + n] = sf[j];
            a.sg[base + (size_t)(p0 + j) * N + n] = sg[j];
        }
    }
    if (threadIdx.x == 0) a.dec[((size_t)b * a.H + h) * a.nc + c] = expf(cl);
}

// Step 2: state entering each chunk (forward pass over chunks) and adjoint entering each chunk
// from the right (reverse pass), both in place.  A (batch, head) pair's P x N entries are split
// over gridDim.z CTAs; a thread owns four neighbouring entries.  The dependent chain over the
// chunks reads its inputs from a ring of kRing chunks in shared memory that asynchronous copies
// fill ahead of it, so that kRing - 1 chunks' loads are always in flight.
constexpr int kPassE = 4;
constexpr int kRing = 12;      // 12 chunks x 256 threads x 16 B = 48 KB of static shared memory

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

template <int P, int N>
__global__ void __launch_bounds__(kT) k_bwd_pass(BwdArgs a) {
    __shared__ __align__(16) float4 ring[kRing][kT];
    const int h = blockIdx.x, b = blockIdx.y;
    const int e = kPassE * (blockIdx.z * kT + threadIdx.x);
    const size_t dbase = ((size_t)b * a.H + h) * a.nc;
    for (int dirn = 0; dirn < 2; ++dirn) {
        // dirn 0: states S (a.sf), chunks in increasing order; dirn 1: adjoints (a.sg), decreasing
        float *arr = dirn == 0 ? a.sf : a.sg;
        auto chunk_of = [&](int i) { return dirn == 0 ? i : a.nc - 1 - i; };
        // one commit group per chunk index (empty past the last chunk), into ring slot i % kRing
        auto issue = [&](int i, int slot) {
            if (i < a.nc) cp_async16(&ring[slot][threadIdx.x], arr + chunk_slot(a, b, h, chunk_of(i), P * N) + e);
            cp_async_commit();
        };
#pragma unroll
        for (int u = 0; u < kRing - 1; ++u) issue(u, u);
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = 0; i0 < a.nc; i0 += kRing) {
            float dcb[kRing];
#pragma unroll
            for (int u = 0; u < kRing; ++u) dcb[u] = i0 + u < a.nc ? a.dec[dbase + chunk_of(i0 + u)] : 0.f;
#pragma unroll
            for (int u = 0; u < kRing; ++u) {
                const int i = i0 + u;
                if (i >= a.nc) break;
                issue(i + kRing - 1, (u + kRing - 1) % kRing);
                cp_async_wait<kRing - 1>();              // chunk i has landed in slot u
                const float4 v = ring[u][threadIdx.x];
                *reinterpret_cast<float4 *>(arr + chunk_slot(a, b, h, chunk_of(i), P * N) + e) = r;
                r.x = fmaf(dcb[u], r.x, v.x);
                r.y = fmaf(dcb[u], r.y, v.y);
                r.z = fmaf(dcb[u], r.z, v.z);
                r.w = fmaf(dcb[u], r.w, v.w);
            }
        }
        cp_async_wait<0>();                              // the ring is reused by the next pass
    }
}

// Step 2 for small states (P N < kT kPassE): one entry per thread or fewer.
template <int P, int N>
__global__ void __launch_bounds__(kT) k_bwd_pass_small(BwdArgs a) {
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t base = ((size_t)b * a.H + h) * a.nc;
    for (int e = threadIdx.x; e < P * N; e += kT) {
        float run = 0.f;
        for (int c = 0; c < a.nc; ++c) {
            float *S = a.sf + chunk_slot(a, b, h, c, P * N);
            const float v = S[e];
            S[e] = run;
            run = fmaf(a.dec[base + c], run, v);
        }
        run = 0.f;
        for (int c = a.nc - 1; c >= 0; --c) {
            float *Z = a.sg + chunk_slot(a, b, h, c, P * N);
            const float v = Z[e];
            Z[e] = run;
            run = fmaf(a.dec[base + c], run, v);
        }
    }
}

// Step 3: every per-position gradient of one chunk.  Pair terms (k, s) inside the chunk use
// E[k][s] = (C_k . B_s) exp(cs_k - cs_s) for s <= k (else 0) and
// F[k][s] = (x_k . gy_s) exp(cs_s - cs_k) for s >= k (else 0); the entering state Sin and the
// entering adjoint Gin carry everything outside the chunk.  The forward output is not
// recomputed: <gy_k, y_k - D x_k> = exp(cs_k) C_k . (Sin gy_k) + sum_{s<=k} E[k][s] dt_s x_s . gy_k,
// whose first part falls out of the dC products.  Every product below is a small matrix product
// evaluated in register tiles (2 or 4 k and 8 columns per thread), so that each shared-memory
// load feeds several multiply-adds.
constexpr int kQm = 64;        // largest chunk of the gradient kernels
constexpr int kSQ = kQm + 1;   // row stride of E and F (odd: column reads hit distinct banks)

template <int P, int N>
struct ChunkSmem {
    static constexpr int SX = P + 4;   // rows of x, gy (16-byte aligned, 4 banks apart)
    static constexpr int SB = N + 4;   // rows of B, C and of Sin, Gin in [p][n] order
    // one of Sin, Gin in either order; also the [k][p] hand-off of the two CTA halves
    static constexpr int kS2 = (N * SX > P * SB) ? N * SX : P * SB;
    static constexpr int kS = kS2 > kQm * P ? kS2 : kQm * P;
    static constexpr int kCs = 0, kDt = 64, kRed = 128, kX = 320, kGy = kX + kQm * SX, kB = kGy + kQm * SX,
                         kC = kB + kQm * SB, kS0 = kC + kQm * SB, kS1 = kS0 + kS, kE = kS1 + kS, kF = kE + kQm * kSQ,
                         kFloats = kF + kQm * kSQ;
};

// acc[j] += m v[col(j)] over a thread's eight columns col(j) = (j & 3) + (j >> 2) HALF: two groups
// of four, HALF apart.  The lanes of a warp take consecutive groups of four, so each 16-byte
// load of a warp reads one contiguous run of the row (no bank conflicts).
template <int HALF>
__device__ __forceinline__ void fma8(float (&acc)[8], float m, const float *v) {
    const float4 a = *reinterpret_cast<const float4 *>(v), b = *reinterpret_cast<const float4 *>(v + HALF);
    acc[0] = fmaf(m, a.x, acc[0]); acc[1] = fmaf(m, a.y, acc[1]); acc[2] = fmaf(m, a.z, acc[2]);
    acc[3] = fmaf(m, a.w, acc[3]); acc[4] = fmaf(m, b.x, acc[4]); acc[5] = fmaf(m, b.y, acc[5]);
    acc[6] = fmaf(m, b.z, acc[6]); acc[7] = fmaf(m, b.w, acc[7]);
}

template <typename T, int P, int N>
__global__ void __launch_bounds__(kTC) k_bwd_chunk(BwdArgs a) {
    using L_ = ChunkSmem<P, N>;
    constexpr int SX = L_::SX, SB = L_::SB;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int Q = a.Q, g = h / (a.H / a.G);
    const int tid = threadIdx.x;
    extern __shared__ __align__(16) float sm[];
    float *cs = sm + L_::kCs, *dts = sm + L_::kDt, *red = sm + L_::kRed;   // red: [3][64] u, <gy, y - D x>, <gy, x>
    float *xs = sm + L_::kX, *gys = sm + L_::kGy, *bs = sm + L_::kB, *cc = sm + L_::kC;
    float *S0 = sm + L_::kS0, *S1 = sm + L_::kS1, *E = sm + L_::kE, *F = sm + L_::kF;
    auto xrow = [&](int k) { return (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.H + h) * P; };
    auto brow = [&](int k) { return (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.G + g) * N; };
    load_rows2<T, N, kTC>(Q, (const T *)a.B, (const T *)a.C, brow,
                          [&](int k, int n, const float (&vb)[8], const float (&vc)[8]) {
                              st8(bs + k * SB + n, vb);
                              st8(cc + k * SB + n, vc);
                          });
    load_rows2<T, P, kTC>(Q, (const T *)a.x, (const T *)a.gy, xrow,
                          [&](int k, int p, const float (&vx)[8], const float (&vg)[8]) {
                              st8(xs + k * SX + p, vx);
                              st8(gys + k * SX + p, vg);
                          });
    bwd_cumsum<T>(a, b, h, c, cs, dts);
    const float cl = cs[Q - 1];
    // the entering adjoint in [n][p] order for the (k, p) outputs: a lane reads four n of one p,
    // and the lanes of a warp take consecutive p, so the stores hit distinct banks
    const size_t sbase = chunk_slot(a, b, h, c, P * N);
    constexpr int kSU = (P * N / 4 + kTC - 1) / kTC;
    {
        float4 gv[kSU];
#pragma unroll
        for (int u = 0; u < kSU; ++u) {
            const int i = tid + kTC * u;
            if (i < P * (N / 4)) {
                const int p = i % P, n = 4 * (i / P);
                gv[u] = *reinterpret_cast<const float4 *>(a.sg + sbase + (size_t)p * N + n);
            }
        }
#pragma unroll
        for (int u = 0; u < kSU; ++u) {
            const int i = tid + kTC * u;
            if (i < P * (N / 4)) {
                const int p = i % P, n = 4 * (i / P);
                S0[n * SX + p] = gv[u].x; S0[(n + 1) * SX + p] = gv[u].y;
                S0[(n + 2) * SX + p] = gv[u].z; S0[(n + 3) * SX + p] = gv[u].w;
            }
        }
    }
    for (int i = tid; i < 3 * 64; i += kTC) red[i] = 0.f;
    __syncthreads();

    // E (threads 0..255) and F (threads 256..511), 4 x 4 tiles.  For Q = 64 a warp covers
    // 32 k x 16 s with k = k0 + 8i, s = s0 + 4j, so the rows read by one instruction are
    // consecutive and their 16-byte pieces fall in distinct banks.
    {
        const bool second = tid >= kTC / 2;
        const int t = tid & (kTC / 2 - 1);
        const int qt = Q / 4;
        if (t < qt * qt) {
            int k0, kst, s0, sst;
            if (Q == kQm) {
                const int w = t >> 5, l = t & 31;
                k0 = 32 * (w & 1) + (l & 7); kst = 8; s0 = 16 * (w >> 1) + (l >> 3); sst = 4;
            } else {
                k0 = 4 * (t % qt); kst = 1; s0 = 4 * (t / qt); sst = 1;
            }
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
            const float *ra = second ? xs : cc, *rb = second ? gys : bs;
            const int st = second ? SX : SB, K = second ? P : N;
            // four K steps per iteration: each row is read as one 16-byte vector
#pragma unroll 2
            for (int kk = 0; kk < K; kk += 4) {
                float4 av[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = *reinterpret_cast<const float4 *>(ra + (k0 + kst * i) * st + kk);
#pragma unroll
                for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4 *>(rb + (s0 + sst * j) * st + kk);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[i][j] = fmaf(av[i].x, bv[j].x, acc[i][j]);
                        acc[i][j] = fmaf(av[i].y, bv[j].y, acc[i][j]);
                        acc[i][j] = fmaf(av[i].z, bv[j].z, acc[i][j]);
                        acc[i][j] = fmaf(av[i].w, bv[j].w, acc[i][j]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = k0 + kst * i, s = s0 + sst * j;
                    if (!second) E[k * kSQ + s] = s <= k ? acc[i][j] * expf(cs[k] - cs[s]) : 0.f;
                    else F[k * kSQ + s] = s >= k ? acc[i][j] * expf(cs[s] - cs[k]) : 0.f;
                }
        }
    }
    __syncthreads();

    // <gy_k, y_k - D x_k> without y: its intra-chunk part is sum_{s <= k} E[k][s] dt_s (x_s . gy_k)
    // with x_s . gy_k = F[s][k] exp(cs_s - cs_k) (the entering-state part is added with the dC
    // products below), and <gy_k, x_k> = F[k][k].  Eight lanes per position.
    {
        const int k = tid >> 3, sl = tid & 7;
        float acc = 0.f;
        if (k < Q) {
            for (int s = sl; s <= k; s += 8) {
                const float d = cs[s] - cs[k];           // >= 0; F[s][k] carries exp(-d)
                if (d < 80.f) acc = fmaf(E[k * kSQ + s] * dts[s], F[s * kSQ + k] * expf(d), acc);
            }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        if (k < Q && sl == 0) {
            red[64 + k] = acc;
            red[128 + k] = F[k * kSQ + k];
        }
    }

    // outputs over (k, p): the adjoint times B (its entering part and the chunk's own part) and
    // dx.  Thread: rows k0, k0 + 1 and columns p0 + (j & 3) + (j >> 2) P/2.  The two halves of the CTA take
    // alternate s of the chunk's own part and one half each of the state index n of the entering
    // part; the second half hands its sums to the first through the entering state's buffer
    // (not loaded yet).  The PG threads of one row pair are consecutive lanes.
    constexpr int PG = P / 8;
    {
        const float dh = a.D ? a.D[h] : 0.f;
        const int half = tid >= kTC / 2;               // uniform per warp
        const int t = tid & (kTC / 2 - 1);
        const bool active = t < (Q / 2) * PG;
        constexpr int HP = P / 2;
        const int k0 = 2 * (t / PG), p0 = 4 * (t % PG);
        float *xch = S1;                               // [k][p], Q P floats
        float g0[8], g1[8];
        if (active) {
            float gb0[8], gb1[8], go0[8], go1[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) gb0[j] = gb1[j] = go0[j] = go1[j] = 0.f;
            // E[k0][k0 + 1] is 0
            for (int s = k0 + half; s < Q; s += 2) {
                const float *v = gys + s * SX + p0;
                fma8<HP>(gb0, E[s * kSQ + k0], v);
                fma8<HP>(gb1, E[s * kSQ + k0 + 1], v);
            }
            const int n1 = half * (N / 2);
#pragma unroll 4
            for (int n = n1; n < n1 + N / 2; ++n) {
                const float *v = S0 + n * SX + p0;
                fma8<HP>(go0, bs[k0 * SB + n], v);
                fma8<HP>(go1, bs[(k0 + 1) * SB + n], v);
            }
            const float el0 = expf(cl - cs[k0]), el1 = expf(cl - cs[k0 + 1]);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                g0[j] = fmaf(el0, go0[j], gb0[j]);
                g1[j] = fmaf(el1, go1[j], gb1[j]);
            }
            if (half) {
                st8<HP>(xch + k0 * P + p0, g0);
                st8<HP>(xch + (k0 + 1) * P + p0, g1);
            }
        }
        __syncthreads();
        if (!half) {
            float r0a = 0.f, r0b = 0.f;
            if (active) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int k = k0 + kk;
                    const float *gk = kk ? g1 : g0;
                    float gxo[8], r0 = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int pj = p0 + (j & 3) + (j >> 2) * HP;
                        const float g_ = gk[j] + xch[k * P + pj];
                        gxo[j] = fmaf(dts[k], g_, dh * gys[k * SX + pj]);
                        r0 = fmaf(xs[k * SX + pj], g_, r0);
                    }
                    if (kk) r0b = r0; else r0a = r0;
                    const int tk = tok(c * Q + k, a.L, a.dir);
                    float *gxp = a.gx + (((size_t)b * a.L + tk) * a.H + h) * P + p0;
                    *reinterpret_cast<float4 *>(gxp) = make_float4(gxo[0], gxo[1], gxo[2], gxo[3]);
                    *reinterpret_cast<float4 *>(gxp + HP) = make_float4(gxo[4], gxo[5], gxo[6], gxo[7]);
                }
            }
#pragma unroll
            for (int o = PG / 2; o > 0; o >>= 1) {
                r0a += __shfl_xor_sync(0xffffffffu, r0a, o);
                r0b += __shfl_xor_sync(0xffffffffu, r0b, o);
            }
            if (active && (t & (PG - 1)) == 0) {
                red[k0] = r0a;
                red[k0 + 1] = r0b;
            }
        }
    }
    __syncthreads();
    // the entering adjoint again, now in [p][n] order, and the entering state in [p][n] order
    {
        float4 gv[kSU], sv[kSU];
#pragma unroll
        for (int u = 0; u < kSU; ++u) {
            const int i = tid + kTC * u;
            if (i < P * (N / 4)) {
                gv[u] = *reinterpret_cast<const float4 *>(a.sg + sbase + 4 * (size_t)i);
                sv[u] = *reinterpret_cast<const float4 *>(a.sf + sbase + 4 * (size_t)i);
            }
        }
#pragma unroll
        for (int u = 0; u < kSU; ++u) {
            const int i = tid + kTC * u;
            if (i < P * (N / 4)) {
                const int o = (i / (N / 4)) * SB + 4 * (i % (N / 4));
                *reinterpret_cast<float4 *>(S0 + o) = gv[u];
                *reinterpret_cast<float4 *>(S1 + o) = sv[u];
            }
        }
    }
    __syncthreads();

    // outputs over (k, n): this head's parts of dB (threads 0 .. kTC/2 - 1) and of dC (the
    // rest).  Thread: rows k0 .. k0 + 3 and columns n0 + (j & 3) + (j >> 2) N/2; the NG threads
    // of one row quad are consecutive lanes.
    constexpr int NG = N / 8;
    {
        const bool second = tid >= kTC / 2;            // uniform per warp
        const int t = tid & (kTC / 2 - 1);
        const bool active = t < (Q / 4) * NG;
        constexpr int HN = N / 2;
        const int k0 = 4 * (t / NG), n0 = 4 * (t % NG);
        float acc[4][8], pro[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = pro[i][j] = 0.f;
        if (active && !second) {
            // sum over s >= k of F[k][s] C_s (F[k][s] = 0 for s < k); x_k . Gin
            for (int s = k0; s < Q; ++s) {
                const float *cv = cc + s * SB + n0;
#pragma unroll
                for (int i = 0; i < 4; ++i) fma8<HN>(acc[i], F[(k0 + i) * kSQ + s], cv);
            }
#pragma unroll 2
            for (int p = 0; p < P; ++p) {
                const float *gi = S0 + p * SB + n0;
#pragma unroll
                for (int i = 0; i < 4; ++i) fma8<HN>(pro[i], xs[(k0 + i) * SX + p], gi);
            }
        } else if (active) {
            // sum over s <= k of F[s][k] dt_s B_s (F[s][k] = 0 for s > k); gy_k . Sin
            for (int s = 0; s <= k0 + 3; ++s) {
                const float d = dts[s];
                const float *bv = bs + s * SB + n0;
#pragma unroll
                for (int i = 0; i < 4; ++i) fma8<HN>(acc[i], F[s * kSQ + k0 + i] * d, bv);
            }
#pragma unroll 2
            for (int p = 0; p < P; ++p) {
                const float *si = S1 + p * SB + n0;
#pragma unroll
                for (int i = 0; i < 4; ++i) fma8<HN>(pro[i], gys[(k0 + i) * SX + p], si);
            }
        }
        float rpart[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int k = k0 + i;
                const float ek = expf(cs[k]), el = expf(cl - cs[k]), dk = dts[k];
                float o[8];
                if (!second) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = dk * fmaf(el, pro[i][j], acc[i][j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        o[j] = fmaf(ek, pro[i][j], acc[i][j]);
                        rpart[i] = fmaf(cc[k * SB + n0 + (j & 3) + (j >> 2) * HN], pro[i][j], rpart[i]);   // C_k . (Sin gy_k)
                    }
                    rpart[i] *= ek;
                }
                const int tk = tok(c * Q + k, a.L, a.dir);
                float *op = (second ? a.gCh : a.gBh) + (((size_t)b * a.L + tk) * a.H + h) * N + n0;
                *reinterpret_cast<float4 *>(op) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4 *>(op + HN) = make_float4(o[4], o[5], o[6], o[7]);
            }
        }
        if (second) {
#pragma unroll
            for (int o = NG / 2; o > 0; o >>= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i) rpart[i] += __shfl_xor_sync(0xffffffffu, rpart[i], o);
            if (active && (t & (NG - 1)) == 0)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[64 + k0 + i] += rpart[i];
        }
    }
    __syncthreads();
    for (int k = tid; k < Q; k += kTC) {
        const int tk = tok(c * Q + k, a.L, a.dir);
        const size_t ti = ((size_t)b * a.L + tk) * a.H + h;
        a.u[ti] = red[k];
        a.gcs[ti] = red[64 + k] - dts[k] * red[k];
    }
    if (tid == 0) {
        float sx = 0.f;
        for (int k = 0; k < Q; ++k) sx += red[128 + k];
        a.gxd[((size_t)b * a.H + h) * a.nc + c] = sx;
    }
}

// Step 4: ddt and the per-sequence parts of dA and dD, walking the sequence from its last scan
// position in tiles of kT positions (suffix sums of gcs carried across tiles).
template <typename T>
__global__ void __launch_bounds__(kT) k_bwd_dt(BwdArgs a) {
    __shared__ float wsum[kT / 32];
    __shared__ float acc_s[kT / 32];
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float Ah = a.A[h];
    float carry = 0.f, gA = 0.f;
    for (int k1 = a.L; k1 > 0; k1 -= kT) {
        // position k = k1 - 1 - tid: the tile's suffix sums run from high k to low k, i.e. a
        // prefix sum over tid
        const int k = k1 - 1 - tid;
        float v = 0.f, dtv = 0.f, uv = 0.f;
        size_t ti = 0;
        if (k >= 0) {
            const int t = tok(k, a.L, a.dir);
            ti = ((size_t)b * a.L + t) * a.H + h;
            v = a.gcs[ti];
            uv = a.u[ti];
            dtv = ldf<T>((const T *)a.dt, ti);
        }
        float s = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float w = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += w;
        }
        if (lane == 31) wsum[warp] = s;
        __syncthreads();
        float base = carry;
        for (int w = 0; w < warp; ++w) base += wsum[w];
        const float suf = base + s;                  // sum of gcs over positions >= k
        if (k >= 0) {
            a.gdt[ti] = fmaf(Ah, suf, uv);
            gA = fmaf(dtv, suf, gA);
        }
        float tile = 0.f;
        for (int w = 0; w < kT / 32; ++w) tile += wsum[w];
        carry += tile;
        __syncthreads();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gA += __shfl_xor_sync(0xffffffffu, gA, o);
    if (lane == 0) acc_s[warp] = gA;
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kT / 32; ++w) t += acc_s[w];
        a.gAp[(size_t)b * a.H + h] = t;
        float d = 0.f;
        for (int c = 0; c < a.nc; ++c) d += a.gxd[((size_t)b * a.H + h) * a.nc + c];
        a.gDp[(size_t)b * a.H + h] = d;
    }
}

// Step 5: dB, dC summed over the heads of each group (unless the per-chunk kernel summed them
// already: gBh null); dA, dD summed over the batch.
__global__ void __launch_bounds__(kT) k_bwd_reduce(BwdArgs a) {
    const size_t total = a.gBh ? (size_t)a.batch * a.L * a.G * a.N : 0;
    const int per = a.H / a.G;
    for (size_t i = (size_t)blockIdx.x * kT + threadIdx.x; i < total; i += (size_t)gridDim.x * kT) {
        const int n = (int)(i % a.N);
        const size_t r = i / a.N;                 // (b * L + t) * G + g
        const int g = (int)(r % a.G);
        const size_t bt = r / a.G;
        float sb = 0.f, sc = 0.f;
        for (int hh = 0; hh < per; ++hh) {
            const size_t hi = (bt * a.H + (size_t)g * per + hh) * a.N + n;
            sb += a.gBh[hi];
            sc += a.gCh[hi];
        }
        a.gB[i] = sb;
        a.gC[i] = sc;
    }
    if (blockIdx.x == 0) {
        for (int h = threadIdx.x; h < a.H; h += kT) {
            float sa = 0.f, sd = 0.f;
            for (int b = 0; b < a.batch; ++b) {
                sa += a.gAp[(size_t)b * a.H + h];
                sd += a.gDp[(size_t)b * a.H + h];
            }
            a.gA[h] = sa;
            if (a.gD) a.gD[h] = sd;
        }
    }
}

template <typename T, int P, int N>
cudaError_t bwd_typed(const BwdArgs &a, cudaStream_t st) {
    const int Q = a.Q;
    // 128-position chunks of the tensor-core shape: chunk sums and per-chunk gradients on tcgen05
    const bool tc = Q == 128 && bwd_tc_supported(a, sizeof(T) == 2);
    if (Q > kQm && !tc) return cudaErrorInvalidValue;
    const size_t sm1 = sizeof(float) * (128 + 2 * Q * P + 2 * Q * N);
    const size_t sm3 = sizeof(float) * ChunkSmem<P, N>::kFloats;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_sums<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_bwd_chunk<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
    if (e != cudaSuccess) return e;
    if (tc) {
        if ((e = launch_bwd_tc_sums(a, st)) != cudaSuccess) return e;
    } else {
        k_bwd_chunk_sums<T, P, N><<<dim3(a.nc, a.H, a.batch), kT, sm1, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    static_assert(P * N % (kT * kPassE) == 0 || P * N < kT * kPassE, "pass slicing");
    if constexpr (P * N >= kT * kPassE) {
        k_bwd_pass<P, N><<<dim3(a.H, a.batch, P * N / (kT * kPassE)), kT, 0, st>>>(a);
    } else {
        k_bwd_pass_small<P, N><<<dim3(a.H, a.batch), kT, 0, st>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    BwdArgs ar = a;
    if (tc) {
        if ((e = launch_bwd_tc_chunk(a, st)) != cudaSuccess) return e;
        ar.gBh = ar.gCh = nullptr;             // dB, dC already summed over the heads
    } else {
        k_bwd_chunk<T, P, N><<<dim3(a.nc, a.H, a.batch), kTC, sm3, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_bwd_dt<T><<<dim3(a.H, a.batch), kT, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t total = ar.gBh ? (size_t)a.batch * a.L * a.G * a.N : 0;
    const int blocks = (int)((total + kT - 1) / kT < 148 * 8 ? (total + kT - 1) / kT : 148 * 8);
    k_bwd_reduce<<<blocks > 0 ? blocks : 1, kT, 0, st>>>(ar);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_dtype(const BwdArgs &a, cudaStream_t st) {
#define SSD_BWD_CASE(PP, NN) if (a.P == PP && a.N == NN) return bwd_typed<T, PP, NN>(a, st);
    SSD_BWD_CASE(16, 16) SSD_BWD_CASE(16, 32) SSD_BWD_CASE(16, 64) SSD_BWD_CASE(16, 128)
    SSD_BWD_CASE(32, 16) SSD_BWD_CASE(32, 32) SSD_BWD_CASE(32, 64) SSD_BWD_CASE(32, 128)
    SSD_BWD_CASE(64, 16) SSD_BWD_CASE(64, 32) SSD_BWD_CASE(64, 64) SSD_BWD_CASE(64, 128)
#undef SSD_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_bwd(const BwdArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? bwd_dtype<__nv_bfloat16>(a, st) : bwd_dtype<float>(a, st);
}

}  // namespace ssd
