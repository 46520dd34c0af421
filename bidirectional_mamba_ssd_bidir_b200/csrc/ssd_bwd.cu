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
    extern __shared__ float sm[];
    float *cs = sm, *dts = cs + 64, *xw = dts + 64, *gw = xw + Q * P, *bs = gw + Q * P, *cc = bs + Q * N;
    bwd_cumsum<T>(a, b, h, c, cs, dts);
    const float cl = cs[Q - 1];
    for (int i = threadIdx.x; i < Q * P; i += kT) {
        const int k = i / P, p = i % P;
        const size_t xi = (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.H + h) * P + p;
        xw[i] = expf(cl - cs[k]) * dts[k] * ldf<T>((const T *)a.x, xi);
        gw[i] = expf(cs[k]) * ldf<T>((const T *)a.gy, xi);
    }
    for (int i = threadIdx.x; i < Q * N; i += kT) {
        const int k = i / N, n = i % N;
        const size_t bi = (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.G + g) * N + n;
        bs[i] = ldf<T>((const T *)a.B, bi);
        cc[i] = ldf<T>((const T *)a.C, bi);
    }
    __syncthreads();
    float sf[E], sg[E];
#pragma unroll
    for (int j = 0; j < E; ++j) sf[j] = sg[j] = 0.f;
    const int n = threadIdx.x % N;
    for (int k = 0; k < Q; ++k) {
        const float bv = bs[k * N + n], cv = cc[k * N + n];
#pragma unroll
        for (int j = 0; j < E; ++j) {
            const int p = (threadIdx.x + kT * j) / N;
            sf[j] = fmaf(xw[k * P + p], bv, sf[j]);
            sg[j] = fmaf(gw[k * P + p], cv, sg[j]);
        }
    }
    const size_t base = (((size_t)b * a.H + h) * a.nc + c) * P * N;
#pragma unroll
    for (int j = 0; j < E; ++j) {
        a.sf[base + threadIdx.x + kT * j] = sf[j];
        a.sg[base + threadIdx.x + kT * j] = sg[j];
    }
    if (threadIdx.x == 0) a.dec[((size_t)b * a.H + h) * a.nc + c] = expf(cl);
}

// Step 2: state entering each chunk (forward pass over chunks) and adjoint entering each chunk
// from the right (reverse pass), both in place.  A (batch, head) pair's P x N entries are split
// over gridDim.z CTAs of kPassE entries per thread; each chunk's values are loaded before any
// of them is overwritten, so the loads of one chunk overlap.
constexpr int kPassE = 2;
template <int P, int N>
__global__ void __launch_bounds__(kT) k_bwd_pass(BwdArgs a) {
    const int h = blockIdx.x, b = blockIdx.y;
    const int e0 = blockIdx.z * kT * kPassE + threadIdx.x;
    const size_t base = ((size_t)b * a.H + h) * a.nc;
    float run[kPassE], v[kPassE];
#pragma unroll
    for (int j = 0; j < kPassE; ++j) run[j] = 0.f;
    for (int c = 0; c < a.nc; ++c) {
        float *S = a.sf + (base + c) * P * N;
        const float dc = a.dec[base + c];
#pragma unroll
        for (int j = 0; j < kPassE; ++j) v[j] = S[e0 + kT * j];
#pragma unroll
        for (int j = 0; j < kPassE; ++j) {
            S[e0 + kT * j] = run[j];
            run[j] = fmaf(dc, run[j], v[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < kPassE; ++j) run[j] = 0.f;
    for (int c = a.nc - 1; c >= 0; --c) {
        float *Z = a.sg + (base + c) * P * N;
        const float dc = a.dec[base + c];
#pragma unroll
        for (int j = 0; j < kPassE; ++j) v[j] = Z[e0 + kT * j];
#pragma unroll
        for (int j = 0; j < kPassE; ++j) {
            Z[e0 + kT * j] = run[j];
            run[j] = fmaf(dc, run[j], v[j]);
        }
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
            float *S = a.sf + (base + c) * P * N;
            const float v = S[e];
            S[e] = run;
            run = fmaf(a.dec[base + c], run, v);
        }
        run = 0.f;
        for (int c = a.nc - 1; c >= 0; --c) {
            float *Z = a.sg + (base + c) * P * N;
            const float v = Z[e];
            Z[e] = run;
            run = fmaf(a.dec[base + c], run, v);
        }
    }
}

// Step 3: every per-position gradient of one chunk.  Pair terms (k, s) inside the chunk use
// CB[k][s] = C_k . B_s, XG[k][s] = x_k . gy_s and Lm[k][s] = exp(cs_k - cs_s) (s <= k, else 0);
// the entering state Sin and the entering adjoint Gin carry everything outside the chunk.
template <typename T, int P, int N>
__global__ void __launch_bounds__(kTC) k_bwd_chunk(BwdArgs a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int Q = a.Q, g = h / (a.H / a.G);
    // rows of x, gy (stride P + 1), B, C (stride N + 1) and of the entering state and adjoint
    // (stride N + 1) are padded by one word, so that a warp reading one column across rows hits
    // 32 different banks
    constexpr int SP = P + 1, SN = N + 1;
    extern __shared__ float sm[];
    float *cs = sm, *dts = cs + 64, *xs = dts + 64, *gys = xs + Q * SP, *bs = gys + Q * SP, *cc = bs + Q * SN;
    float *CB = cc + Q * SN, *XG = CB + Q * Q, *Lm = XG + Q * Q, *Sin = Lm + Q * Q, *Gin = Sin + P * SN;
    float *red = Gin + P * SN;   // [3][64]: u, <gy, y - D x>, <gy, x> per position
    bwd_cumsum<T>(a, b, h, c, cs, dts);
    const float cl = cs[Q - 1];
    for (int i = threadIdx.x; i < Q * P; i += kTC) {
        const int k = i / P, p = i % P;
        const size_t xi = (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.H + h) * P + p;
        xs[k * SP + p] = ldf<T>((const T *)a.x, xi);
        gys[k * SP + p] = ldf<T>((const T *)a.gy, xi);
    }
    for (int i = threadIdx.x; i < Q * N; i += kTC) {
        const int k = i / N, n = i % N;
        const size_t bi = (((size_t)b * a.L + tok(c * Q + k, a.L, a.dir)) * a.G + g) * N + n;
        bs[k * SN + n] = ldf<T>((const T *)a.B, bi);
        cc[k * SN + n] = ldf<T>((const T *)a.C, bi);
    }
    const size_t sbase = (((size_t)b * a.H + h) * a.nc + c) * P * N;
    for (int i = threadIdx.x; i < P * N; i += kTC) {
        const int p = i / N, n = i % N;
        Sin[p * SN + n] = a.sf[sbase + i];
        Gin[p * SN + n] = a.sg[sbase + i];
    }
    for (int i = threadIdx.x; i < 3 * 64; i += kTC) red[i] = 0.f;
    __syncthreads();
    for (int i = threadIdx.x; i < Q * Q; i += kTC) {
        const int k = i / Q, s = i % Q;
        float cb = 0.f, xg = 0.f;
        for (int n = 0; n < N; ++n) cb = fmaf(cc[k * SN + n], bs[s * SN + n], cb);
        for (int p = 0; p < P; ++p) xg = fmaf(xs[k * SP + p], gys[s * SP + p], xg);
        CB[i] = cb;
        XG[i] = xg;
        Lm[i] = s <= k ? expf(cs[k] - cs[s]) : 0.f;
    }
    __syncthreads();

    // outputs over (k, p): y - D x (recomputed), G_k B_k, dx.  A thread takes one position k and
    // four columns p0 + kGP j, so the pair terms of k (read once per s) serve four outputs.
    constexpr int kGP = P / 4;                      // threads per position
    const float dh = a.D ? a.D[h] : 0.f;
    for (int i = threadIdx.x; i < Q * kGP; i += kTC) {
        const int k = i / kGP, p0 = i % kGP;
        float yv[4] = {0.f, 0.f, 0.f, 0.f}, gb[4] = {0.f, 0.f, 0.f, 0.f};
        for (int s = 0; s <= k; ++s) {
            const float m = CB[k * Q + s] * Lm[k * Q + s] * dts[s];
#pragma unroll
            for (int j = 0; j < 4; ++j) yv[j] = fmaf(m, xs[s * SP + p0 + kGP * j], yv[j]);
        }
        for (int s = k; s < Q; ++s) {
            const float m = CB[s * Q + k] * Lm[s * Q + k];
#pragma unroll
            for (int j = 0; j < 4; ++j) gb[j] = fmaf(m, gys[s * SP + p0 + kGP * j], gb[j]);
        }
        float yo[4] = {0.f, 0.f, 0.f, 0.f}, go[4] = {0.f, 0.f, 0.f, 0.f};
        for (int n = 0; n < N; ++n) {
            const float cv = cc[k * SN + n], bv = bs[k * SN + n];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                yo[j] = fmaf(cv, Sin[(p0 + kGP * j) * SN + n], yo[j]);
                go[j] = fmaf(bv, Gin[(p0 + kGP * j) * SN + n], go[j]);
            }
        }
        const float ek = expf(cs[k]), el = expf(cl - cs[k]);
        const int t = tok(c * Q + k, a.L, a.dir);
        float r0 = 0.f, r1 = 0.f, r2 = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + kGP * j;
            const float y_ = fmaf(ek, yo[j], yv[j]), g_ = fmaf(el, go[j], gb[j]);
            const float xv = xs[k * SP + p], gv = gys[k * SP + p];
            a.gx[(((size_t)b * a.L + t) * a.H + h) * P + p] = fmaf(dts[k], g_, dh * gv);
            r0 = fmaf(xv, g_, r0);
            r1 = fmaf(gv, y_, r1);
            r2 = fmaf(gv, xv, r2);
        }
        // the kGP consecutive lanes that share position k reduce their terms; one adds them
#pragma unroll
        for (int o = kGP / 2; o > 0; o >>= 1) {
            r0 += __shfl_xor_sync(0xffffffffu, r0, o);
            r1 += __shfl_xor_sync(0xffffffffu, r1, o);
            r2 += __shfl_xor_sync(0xffffffffu, r2, o);
        }
        if ((threadIdx.x & (kGP - 1)) == 0) {
            atomicAdd(&red[k], r0);
            atomicAdd(&red[64 + k], r1);
            atomicAdd(&red[128 + k], r2);
        }
    }
    // outputs over (k, n): this head's parts of dB and dC, four columns n0 + kGN j per thread
    constexpr int kGN = N / 4;
    for (int i = threadIdx.x; i < Q * kGN; i += kTC) {
        const int k = i / kGN, n0 = i % kGN;
        float gbv[4] = {0.f, 0.f, 0.f, 0.f}, gcv[4] = {0.f, 0.f, 0.f, 0.f};
        for (int s = k; s < Q; ++s) {
            const float m = XG[k * Q + s] * Lm[s * Q + k];
#pragma unroll
            for (int j = 0; j < 4; ++j) gbv[j] = fmaf(m, cc[s * SN + n0 + kGN * j], gbv[j]);
        }
        for (int s = 0; s <= k; ++s) {
            const float m = XG[s * Q + k] * Lm[k * Q + s] * dts[s];
#pragma unroll
            for (int j = 0; j < 4; ++j) gcv[j] = fmaf(m, bs[s * SN + n0 + kGN * j], gcv[j]);
        }
        float bo[4] = {0.f, 0.f, 0.f, 0.f}, co[4] = {0.f, 0.f, 0.f, 0.f};
        for (int p = 0; p < P; ++p) {
            const float xv = xs[k * SP + p], gv = gys[k * SP + p];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bo[j] = fmaf(Gin[p * SN + n0 + kGN * j], xv, bo[j]);
                co[j] = fmaf(Sin[p * SN + n0 + kGN * j], gv, co[j]);
            }
        }
        const float ek = expf(cs[k]), el = expf(cl - cs[k]);
        const int t = tok(c * Q + k, a.L, a.dir);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const size_t oi = (((size_t)b * a.L + t) * a.H + h) * N + n0 + kGN * j;
            a.gBh[oi] = dts[k] * fmaf(el, bo[j], gbv[j]);
            a.gCh[oi] = fmaf(ek, co[j], gcv[j]);
        }
    }
    __syncthreads();
    for (int k = threadIdx.x; k < Q; k += kTC) {
        const int t = tok(c * Q + k, a.L, a.dir);
        const size_t ti = ((size_t)b * a.L + t) * a.H + h;
        a.u[ti] = red[k];
        a.gcs[ti] = red[64 + k] - dts[k] * red[k];
    }
    if (threadIdx.x == 0) {
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

// Step 5: dB, dC summed over the heads of each group; dA, dD summed over the batch.
__global__ void __launch_bounds__(kT) k_bwd_reduce(BwdArgs a) {
    const size_t total = (size_t)a.batch * a.L * a.G * a.N;
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
    const size_t sm1 = sizeof(float) * (128 + 2 * Q * P + 2 * Q * N);
    const size_t sm3 = sizeof(float) * (128 + 2 * Q * (P + 1) + 2 * Q * (N + 1) + 3 * Q * Q + 2 * P * (N + 1) + 3 * 64);
    cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_sums<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_bwd_chunk<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
    if (e != cudaSuccess) return e;
    k_bwd_chunk_sums<T, P, N><<<dim3(a.nc, a.H, a.batch), kT, sm1, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    static_assert(P * N % (kT * kPassE) == 0 || P * N < kT * kPassE, "pass slicing");
    if constexpr (P * N >= kT * kPassE) {
        k_bwd_pass<P, N><<<dim3(a.H, a.batch, P * N / (kT * kPassE)), kT, 0, st>>>(a);
    } else {
        k_bwd_pass_small<P, N><<<dim3(a.H, a.batch), kT, 0, st>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_chunk<T, P, N><<<dim3(a.nc, a.H, a.batch), kTC, sm3, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_dt<T><<<dim3(a.H, a.batch), kT, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t total = (size_t)a.batch * a.L * a.G * a.N;
    const int blocks = (int)((total + kT - 1) / kT < 148 * 8 ? (total + kT - 1) / kT : 148 * 8);
    k_bwd_reduce<<<blocks > 0 ? blocks : 1, kT, 0, st>>>(a);
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
