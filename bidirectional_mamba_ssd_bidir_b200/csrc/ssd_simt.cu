// ssd_simt.cu -- chunked SSD scan on the CUDA cores (float32 FFMA).
//
// This is the general path: any supported headdim/dstate/chunk, float32 or
// bf16 storage, both directions.  It evaluates the scan in the chunked
// (state-passing) form, exactly as the recurrence
//     S <- exp(dt A) S + dt x (outer) B,   y = C.S + D x
// unrolls over a chunk of Q tokens (cs_k = A * sum_{j<=k in chunk} dt_j):
//     intra-chunk  y_diag[k] = sum_{s<=k} (C_k . B_s) exp(cs_k - cs_s) dt_s x_s
//     chunk state  S_c       = sum_s exp(cs_last - cs_s) dt_s x_s (outer) B_s
//     passing      Sin_0 = 0, Sin_{c+1} = exp(cs_last) Sin_c + S_c
//     from state   y_off[k]  = exp(cs_k) C_k . Sin_c
// in three launches: chunk states (all chunks in parallel), the sequential
// pass over chunks, and the outputs (all chunks in parallel).  A single-chunk
// sequence skips the first two unless a state enters or leaves the call.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 16;    // output rows per CTA in the output kernel
constexpr int kSTile = 32;   // tokens per staged tile

// Inclusive prefix sum of dt over one chunk (scan order), times A, into cs[];
// dts[] receives dt.  Every kernel uses this same routine, so the chunk's
// cumulative decays are bit-identical wherever they are recomputed.
template <typename T>
__device__ void chunk_cumsum(const ScanArgs &a, const T *dt, int b, int h, int c, float *cs, float *dts) {
    __shared__ float warp_tot[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Q = a.Q;
    float v = 0.f;
    if (tid < Q) {
        const int t = tok(c * Q + tid, a.L, a.dir);
        v = ldf<T>(dt, ((size_t)b * a.L + t) * a.H + h);
        dts[tid] = v;
    }
    float s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float u = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += u;
    }
    if (lane == 31) warp_tot[warp] = s;
    __syncthreads();
    float base = 0.f;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    if (tid < Q) cs[tid] = a.A[h] * (base + s);
    __syncthreads();
}

// Offset of the P x N state of (b, h, chunk c) in a.states.  The heads of one chunk are
// neighbours, so the state pass, which walks all heads chunk by chunk, touches one contiguous
// range at a time.
__device__ __forceinline__ size_t state_slot(const ScanArgs &a, int b, int h, int c, int PN) {
    return (((size_t)b * a.nc + c) * a.H + h) * (size_t)PN;
}

template <typename T, int P, int N>
__global__ void __launch_bounds__(kThreads) k_chunk_state(ScanArgs a) {
    constexpr int E = P * N / kThreads;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int Q = a.Q, g = h / (a.H / a.G);
    const T *x = (const T *)a.x, *B = (const T *)a.B;
    extern __shared__ float sm[];
    float *cs = sm, *dts = cs + Q, *xs = dts + Q, *bs = xs + kSTile * P;
    chunk_cumsum<T>(a, (const T *)a.dt, b, h, c, cs, dts);
    const float cl = cs[Q - 1];
    float acc[E];
#pragma unroll
    for (int j = 0; j < E; ++j) acc[j] = 0.f;
    const int n = threadIdx.x % N;
    for (int s0 = 0; s0 < Q; s0 += kSTile) {
        // rows past the chunk end (chunk shorter than a tile) are zero
        for (int i = threadIdx.x; i < kSTile * P; i += kThreads) {
            const int r = i / P, p = i % P, k = s0 + r;
            float v = 0.f;
            if (k < Q) {
                const int t = tok(c * Q + k, a.L, a.dir);
                v = expf(cl - cs[k]) * dts[k] * ldf<T>(x, (((size_t)b * a.L + t) * a.H + h) * P + p);
            }
            xs[i] = v;
        }
        for (int i = threadIdx.x; i < kSTile * N; i += kThreads) {
            const int r = i / N, nn = i % N, k = s0 + r;
            float v = 0.f;
            if (k < Q) {
                const int t = tok(c * Q + k, a.L, a.dir);
                v = ldf<T>(B, (((size_t)b * a.L + t) * a.G + g) * N + nn);
            }
            bs[i] = v;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kSTile; ++r) {
            const float bv = bs[r * N + n];
#pragma unroll
            for (int j = 0; j < E; ++j) {
                const int p = (threadIdx.x + kThreads * j) / N;
                acc[j] = fmaf(xs[r * P + p], bv, acc[j]);
            }
        }
        __syncthreads();
    }
    float *S = a.states + state_slot(a, b, h, c, P * N);
#pragma unroll
    for (int j = 0; j < E; ++j) S[threadIdx.x + kThreads * j] = acc[j];
    if (threadIdx.x == 0) a.decays[((size_t)b * a.H + h) * a.nc + c] = expf(cl);
}

// The sequential pass over chunks.  A (batch, head)'s P x N entries are split over gridDim.z
// CTAs, kSE neighbouring entries per thread.  The dependent chain reads its inputs from a ring
// of kSRing chunks in shared memory that asynchronous copies fill ahead of it, so that
// kSRing - 1 chunks' loads are always in flight.
constexpr int kSRing = 12;

template <int E>
__device__ __forceinline__ void cp_async_e(float *dst, const float *src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    if constexpr (E == 4) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
    } else {
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
    }
}

template <int P, int N>
struct StatePassShape {
    static constexpr int kE = (P * N >= 4 * kThreads) ? 4 : 1;   // entries per thread
    static constexpr int kSlices = (P * N + kThreads * kE - 1) / (kThreads * kE);
};

template <int P, int N>
__global__ void __launch_bounds__(kThreads) k_state_pass(ScanArgs a) {
    constexpr int E = StatePassShape<P, N>::kE;
    __shared__ __align__(16) float ring[kSRing][kThreads * E];
    const int h = blockIdx.x, b = blockIdx.y;
    const int e = E * (blockIdx.z * kThreads + threadIdx.x);   // this thread's first entry
    const bool mine = e < P * N;
    const size_t sbase = ((size_t)b * a.H + h) * P * N;     // [b][h] slot of s_in / s_out
    const size_t dbase = ((size_t)b * a.H + h) * a.nc;
    float run[E];
#pragma unroll
    for (int j = 0; j < E; ++j) run[j] = (a.s_in && mine) ? a.s_in[sbase + e + j] : 0.f;
    // one commit group per chunk (empty past the last chunk), into ring slot c % kSRing
    auto issue = [&](int c, int slot) {
        if (c < a.nc && mine) cp_async_e<E>(&ring[slot][threadIdx.x * E], a.states + state_slot(a, b, h, c, P * N) + e);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int u = 0; u < kSRing - 1; ++u) issue(u, u);
    for (int c0 = 0; c0 < a.nc; c0 += kSRing) {
        float dcb[kSRing];
#pragma unroll
        for (int u = 0; u < kSRing; ++u) dcb[u] = c0 + u < a.nc ? a.decays[dbase + c0 + u] : 0.f;
#pragma unroll
        for (int u = 0; u < kSRing; ++u) {
            const int c = c0 + u;
            if (c >= a.nc) break;
            issue(c + kSRing - 1, (u + kSRing - 1) % kSRing);
            asm volatile("cp.async.wait_group %0;" ::"n"(kSRing - 1) : "memory");   // chunk c has landed
            if (mine) {
                float *S = a.states + state_slot(a, b, h, c, P * N) + e;
#pragma unroll
                for (int j = 0; j < E; ++j) {
                    const float sc = ring[u][threadIdx.x * E + j];
                    S[j] = run[j];                   // state entering chunk c
                    run[j] = fmaf(dcb[u], run[j], sc);
                }
            }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (a.s_out && mine) {
#pragma unroll
        for (int j = 0; j < E; ++j) a.s_out[sbase + e + j] = run[j];
    }
}

template <typename T, int P, int N>
__global__ void __launch_bounds__(kThreads) k_chunk_output(ScanArgs a, int have_state) {
    constexpr int NP = N + 1;                       // padded row stride (bank spread)
    constexpr int EO = kRows * P / kThreads;        // outputs per thread
    constexpr int EG = kRows * kSTile / kThreads;   // decayed-score entries per thread
    const int tiles = a.Q / kRows;
    const int c = blockIdx.x / tiles, k0 = (blockIdx.x % tiles) * kRows;
    const int h = blockIdx.y, b = blockIdx.z;
    const int Q = a.Q, g = h / (a.H / a.G);
    const T *x = (const T *)a.x, *B = (const T *)a.B, *Cm = (const T *)a.C;
    extern __shared__ float sm[];
    float *cs = sm, *dts = cs + Q, *Cs = dts + Q, *Sin = Cs + kRows * N;
    float *Bs = Sin + (have_state ? P * NP : 0), *xs = Bs + kSTile * NP, *Ms = xs + kSTile * P;
    chunk_cumsum<T>(a, (const T *)a.dt, b, h, c, cs, dts);
    for (int i = threadIdx.x; i < kRows * N; i += kThreads) {
        const int r = i / N, n = i % N;
        const int t = tok(c * Q + k0 + r, a.L, a.dir);
        Cs[i] = ldf<T>(Cm, (((size_t)b * a.L + t) * a.G + g) * N + n);
    }
    if (have_state) {
        const float *S = a.states + state_slot(a, b, h, c, P * N);
        for (int i = threadIdx.x; i < P * N; i += kThreads) Sin[(i / N) * NP + (i % N)] = S[i];
    }
    __syncthreads();

    float yv[EO];
#pragma unroll
    for (int j = 0; j < EO; ++j) {
        const int o = threadIdx.x + kThreads * j, r = o / P, p = o % P;
        float acc = 0.f;
        if (have_state) {
#pragma unroll 8
            for (int n = 0; n < N; ++n) acc = fmaf(Cs[r * N + n], Sin[p * NP + n], acc);
            acc *= expf(cs[k0 + r]);
        }
        yv[j] = acc;
    }

    const int send = k0 + kRows;                    // tokens s < send can reach these rows
    for (int s0 = 0; s0 < send; s0 += kSTile) {
        for (int i = threadIdx.x; i < kSTile * N; i += kThreads) {
            const int r = i / N, n = i % N, s = s0 + r;
            float v = 0.f;
            if (s < Q) {
                const int t = tok(c * Q + s, a.L, a.dir);
                v = ldf<T>(B, (((size_t)b * a.L + t) * a.G + g) * N + n);
            }
            Bs[r * NP + n] = v;
        }
        for (int i = threadIdx.x; i < kSTile * P; i += kThreads) {
            const int r = i / P, p = i % P, s = s0 + r;
            float v = 0.f;
            if (s < Q) {
                const int t = tok(c * Q + s, a.L, a.dir);
                v = ldf<T>(x, (((size_t)b * a.L + t) * a.H + h) * P + p);
            }
            xs[i] = v;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < EG; ++j) {
            const int e = threadIdx.x + kThreads * j, r = e / kSTile, sp = e % kSTile;
            const int k = k0 + r, s = s0 + sp;
            float m = 0.f;
            if (s <= k) {
                float d = 0.f;
#pragma unroll 8
                for (int n = 0; n < N; ++n) d = fmaf(Cs[r * N + n], Bs[sp * NP + n], d);
                m = d * expf(cs[k] - cs[s]) * dts[s];
            }
            Ms[r * kSTile + sp] = m;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < EO; ++j) {
            const int o = threadIdx.x + kThreads * j, r = o / P, p = o % P;
            float acc = yv[j];
#pragma unroll 8
            for (int sp = 0; sp < kSTile; ++sp) acc = fmaf(Ms[r * kSTile + sp], xs[sp * P + p], acc);
            yv[j] = acc;
        }
        __syncthreads();
    }

    const float dh = a.D ? a.D[h] : 0.f;
#pragma unroll
    for (int j = 0; j < EO; ++j) {
        const int o = threadIdx.x + kThreads * j, r = o / P, p = o % P;
        const int t = tok(c * Q + k0 + r, a.L, a.dir);
        const size_t idx = (((size_t)b * a.L + t) * a.H + h) * P + p;   // same as [b][t][h*P+p]
        const float v = fmaf(dh, ldf<T>(x, idx), yv[j]);
        T *y = (T *)a.y;
        if (a.mode == OUT_WRITE) {
            stf<T>(y, idx, v);
        } else if (a.mode == OUT_ACCUM) {
            stf<T>(y, idx, ldf<T>(y, idx) + v);
        } else {
            stf<T>(y, idx, fmaf(a.gate, v, ldf<T>((const T *)a.residual, idx)));
        }
    }
}

// ---------------------------------------------------------------- single-chunk calls
// A call whose sequence is one chunk of at most 64 tokens with no state in or out (the R2L
// block of the Bifocal sidecar is one): nothing crosses a chunk, so one CTA per (head, batch
// row) runs its head's whole scan after a single round of global loads (x, B, C as 16-byte
// vectors, dt, and the residual or the output that the result is added to), instead of the
// several dependent load phases of k_chunk_output.  Same arithmetic: the decays by the same
// prefix sum, the scores C_k . B_s e^(cs_k - cs_s) dt_s for s <= k, their product with x,
// D x and the output mode, in float32.
constexpr int kOneQ = 64;    // longest chunk taken

template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &v, float *f);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4 &v, float *f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &v, float *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// shared floats of one CTA: cs, dt, B and C (rows padded to N + 1), x, the masked scores
__host__ __device__ constexpr size_t one_chunk_floats(int Q, int P, int N) {
    return 2 * (size_t)kOneQ + 2 * (size_t)Q * (N + 1) + (size_t)Q * P + (size_t)Q * Q;
}

template <typename T, int P, int N>
__global__ void __launch_bounds__(kThreads) k_one_chunk(ScanArgs a) {
    constexpr int V = 16 / (int)sizeof(T);                        // elements per 16-byte vector
    constexpr int NB = (kOneQ * N / V + kThreads - 1) / kThreads;  // B (and C) vectors per thread, at most
    constexpr int NX = (kOneQ * P / V + kThreads - 1) / kThreads;  // x vectors per thread, at most
    constexpr int H2 = P / 2;                                      // a thread's two outputs: p and p + P/2
    constexpr int NO = (kOneQ * H2 + kThreads - 1) / kThreads;     // output pairs per thread, at most
    constexpr int NP = N + 1;
    __shared__ float warp_tot[kOneQ / 32];
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Q = a.Q, g = h / (a.H / a.G);
    const T *x = (const T *)a.x, *Bm = (const T *)a.B, *Cm = (const T *)a.C;
    extern __shared__ float sm[];
    float *cs = sm, *dts = cs + kOneQ, *Bs = dts + kOneQ, *Cs = Bs + Q * NP, *xs = Cs + Q * NP, *Ms = xs + Q * P;

    // every global load first
    uint4 vb[NB], vc[NB], vx[NX];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        const int i = tid + kThreads * j;
        if (i < Q * (N / V)) {
            const int s = i / (N / V), cv = i % (N / V);
            const size_t off = (((size_t)b * a.L + tok(s, a.L, a.dir)) * a.G + g) * N + cv * V;
            vb[j] = __ldg(reinterpret_cast<const uint4 *>(Bm + off));
            vc[j] = __ldg(reinterpret_cast<const uint4 *>(Cm + off));
        }
    }
#pragma unroll
    for (int j = 0; j < NX; ++j) {
        const int i = tid + kThreads * j;
        if (i < Q * (P / V)) {
            const int s = i / (P / V), cv = i % (P / V);
            const size_t off = (((size_t)b * a.L + tok(s, a.L, a.dir)) * a.H + h) * P + cv * V;
            vx[j] = __ldg(reinterpret_cast<const uint4 *>(x + off));
        }
    }
    float dtv = 0.f;
    if (tid < Q) dtv = ldf<T>((const T *)a.dt, ((size_t)b * a.L + tok(tid, a.L, a.dir)) * a.H + h);
    // what the result is added to: the residual (OUT_GATE) or the output so far (OUT_ACCUM)
    const T *addend = a.mode == OUT_GATE ? (const T *)a.residual : a.mode == OUT_ACCUM ? (const T *)a.y : nullptr;
    float add0[NO], add1[NO];
#pragma unroll
    for (int j = 0; j < NO; ++j) {
        const int o = tid + kThreads * j;
        add0[j] = add1[j] = 0.f;
        if (addend && o < Q * H2) {
            const size_t row = (((size_t)b * a.L + tok(o / H2, a.L, a.dir)) * a.H + h) * P + o % H2;
            add0[j] = ldf<T>(addend, row);
            add1[j] = ldf<T>(addend, row + H2);
        }
    }

    // cs = A * inclusive prefix sum of dt in scan order: warp scans, then the warps in order
    // (the additions of chunk_cumsum, so the same values)
    float sc = dtv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) sc += u;
    }
    if (lane == 31 && warp < kOneQ / 32) warp_tot[warp] = sc;
    if (tid < Q) dts[tid] = dtv;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        const int i = tid + kThreads * j;
        if (i < Q * (N / V)) {
            const int s = i / (N / V), cv = i % (N / V);
            float f[V];
            unpack16<T>(vb[j], f);
#pragma unroll
            for (int e = 0; e < V; ++e) Bs[s * NP + cv * V + e] = f[e];
            unpack16<T>(vc[j], f);
#pragma unroll
            for (int e = 0; e < V; ++e) Cs[s * NP + cv * V + e] = f[e];
        }
    }
#pragma unroll
    for (int j = 0; j < NX; ++j) {
        const int i = tid + kThreads * j;
        if (i < Q * (P / V)) {
            float f[V];
            unpack16<T>(vx[j], f);
#pragma unroll
            for (int e = 0; e < V; ++e) xs[i * V + e] = f[e];
        }
    }
    __syncthreads();
    if (tid < Q) {
        float base = 0.f;
        for (int w = 0; w < warp; ++w) base += warp_tot[w];
        cs[tid] = a.A[h] * (base + sc);
    }
    __syncthreads();

    // decayed scores M[k][s] for the Q (Q + 1) / 2 pairs s <= k only (pair e: row k with
    // k (k + 1) / 2 <= e < (k + 1) (k + 2) / 2, column s = e - k (k + 1) / 2)
    const int npair = Q * (Q + 1) / 2;
#pragma unroll 1
    for (int e = tid; e < npair; e += kThreads) {
        int k = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
        while (k * (k + 1) / 2 > e) --k;
        while ((k + 1) * (k + 2) / 2 <= e) ++k;
        const int s = e - k * (k + 1) / 2;
        float d0 = 0.f, d1 = 0.f;
#pragma unroll 8
        for (int n = 0; n < N; n += 2) {
            d0 = fmaf(Cs[k * NP + n], Bs[s * NP + n], d0);
            d1 = fmaf(Cs[k * NP + n + 1], Bs[s * NP + n + 1], d1);
        }
        Ms[k * Q + s] = (d0 + d1) * expf(cs[k] - cs[s]) * dts[s];
    }
    __syncthreads();

    // y[k][p] = sum_{s <= k} M[k][s] x[s][p] + D x[k][p] for p and p + P/2, then the output mode
    const float dh = a.D ? a.D[h] : 0.f;
    T *y = (T *)a.y;
#pragma unroll
    for (int j = 0; j < NO; ++j) {
        const int o = tid + kThreads * j;
        if (o < Q * H2) {
            const int k = o / H2, p = o % H2;
            float y0 = 0.f, y1 = 0.f;
#pragma unroll 2
            for (int s = 0; s <= k; ++s) {
                const float m = Ms[k * Q + s];
                y0 = fmaf(m, xs[s * P + p], y0);
                y1 = fmaf(m, xs[s * P + p + H2], y1);
            }
            const float v0 = fmaf(dh, xs[k * P + p], y0), v1 = fmaf(dh, xs[k * P + p + H2], y1);
            const size_t idx = (((size_t)b * a.L + tok(k, a.L, a.dir)) * a.H + h) * P + p;
            if (a.mode == OUT_WRITE) {
                stf<T>(y, idx, v0);
                stf<T>(y, idx + H2, v1);
            } else if (a.mode == OUT_ACCUM) {
                stf<T>(y, idx, add0[j] + v0);
                stf<T>(y, idx + H2, add1[j] + v1);
            } else {
                stf<T>(y, idx, fmaf(a.gate, v0, add0[j]));
                stf<T>(y, idx + H2, fmaf(a.gate, v1, add1[j]));
            }
        }
    }
}

template <typename T, int P, int N>
cudaError_t launch_typed(const ScanArgs &a, cudaStream_t st) {
    // the state kernels run whenever a state crosses a chunk or the call boundary
    const bool multi = a.nc > 1 || a.s_in || a.s_out;
    cudaError_t e;
    if (!multi && a.Q <= kOneQ) {
        const size_t bytes = sizeof(float) * one_chunk_floats(a.Q, P, N);
        if (bytes > 48 * 1024) {
            e = cudaFuncSetAttribute(k_one_chunk<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
        }
        k_one_chunk<T, P, N><<<dim3(a.H, a.batch), kThreads, bytes, st>>>(a);
        return cudaGetLastError();
    }
    const size_t sm_state = sizeof(float) * (2 * a.Q + kSTile * P + kSTile * N);
    const size_t sm_out = sizeof(float) * (2 * a.Q + kRows * N + (multi ? P * (N + 1) : 0) +
                                           kSTile * (N + 1) + kSTile * P + kRows * kSTile);
    if (multi) {
        e = cudaFuncSetAttribute(k_chunk_state<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_state);
        if (e != cudaSuccess) return e;
        k_chunk_state<T, P, N><<<dim3(a.nc, a.H, a.batch), kThreads, sm_state, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_state_pass<P, N><<<dim3(a.H, a.batch, StatePassShape<P, N>::kSlices), kThreads, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(k_chunk_output<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out);
    if (e != cudaSuccess) return e;
    k_chunk_output<T, P, N><<<dim3(a.nc * (a.Q / kRows), a.H, a.batch), kThreads, sm_out, st>>>(a, multi ? 1 : 0);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dtype(const ScanArgs &a, cudaStream_t st) {
#define SSD_CASE(PP, NN) if (a.P == PP && a.N == NN) return launch_typed<T, PP, NN>(a, st);
    SSD_CASE(16, 16) SSD_CASE(16, 32) SSD_CASE(16, 64) SSD_CASE(16, 128)
    SSD_CASE(32, 16) SSD_CASE(32, 32) SSD_CASE(32, 64) SSD_CASE(32, 128)
    SSD_CASE(64, 16) SSD_CASE(64, 32) SSD_CASE(64, 64) SSD_CASE(64, 128)
#undef SSD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_scan(const ScanArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_dtype<__nv_bfloat16>(a, st) : launch_dtype<float>(a, st);
}

}  // namespace ssd
