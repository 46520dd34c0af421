// ssd_internal.cuh -- definitions shared by the launch layer and the kernels.
//
// Notation used throughout the kernels: k is a position in SCAN order
// (0..L-1).  The forward scan reads token t = k; the reverse scan reads token
// t = L-1-k.  Doing every computation in scan order and mapping only the
// addresses is the "flip, scan, flip back" of the R2LM right-to-left stream
// ("Bifocal Diffusion Language Models", section 2, mechanism) without
// materialising a flipped copy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

enum OutMode : int {
    OUT_WRITE = 0,   // y = value
    OUT_ACCUM = 1,   // y = y + value   (second direction of the bidirectional mixer)
    OUT_GATE = 2     // out = residual + gate * value   (R2L sidecar, gate != 0)
};

struct ScanArgs {
    int batch, L, H, P, N, G, Q, nc;
    int dir;                 // +1 forward, -1 reverse
    const void *x, *dt, *B, *C;
    const float *A, *D;      // D may be null
    void *y;                 // output (y, or out for OUT_GATE)
    const void *residual;    // OUT_GATE only
    float gate;              // OUT_GATE only
    int mode;
    float *states;           // [batch][H][nc][P][N] chunk states -> incoming states
    float *decays;           // [batch][H][nc] chunk decay exp(cs_last)
    const float *s_in;       // [batch][H][P][N] state before the first scanned token, or null (zero)
    float *s_out;            // [batch][H][P][N] state after the last scanned token, or null
};

// token index in memory for scan position k
__device__ __forceinline__ int tok(int k, int L, int dir) { return dir > 0 ? k : L - 1 - k; }

template <typename T> __device__ __forceinline__ float ldf(const T *p, size_t i);
template <> __device__ __forceinline__ float ldf<float>(const float *p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void stf(T *p, size_t i, float v);
template <> __device__ __forceinline__ void stf<float>(float *p, size_t i, float v) { p[i] = v; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

// Gradients of one direction of the scan (ssd_bwd.cu).  Inputs in the io
// dtype, gradients and every intermediate in float32.
struct BwdArgs {
    int batch, L, H, P, N, G, Q, nc;
    int dir;
    const void *x, *dt, *B, *C, *gy;
    const float *A, *D;      // D may be null
    float *gx, *gdt, *gA, *gB, *gC, *gD;   // gD may be null
    // workspace
    float *sf;               // [batch][H][nc][P][N] chunk states -> state entering each chunk
    float *sg;               // [batch][H][nc][P][N] adjoint chunk terms -> adjoint entering from the right
    float *dec;              // [batch][H][nc] decay across each chunk
    float *gBh, *gCh;        // [batch][L][H][N] per-head parts of dB and dC
    float *gcs, *u;          // [batch][L][H] dL/dcs and <G_k, x_k B_k^T> per token
    float *gxd;              // [batch][H][nc] per-chunk sum of <gy, x>
    float *gAp, *gDp;        // [batch][H] per-sequence parts of dA and dD
    int *status;             // workspace status word (bounded waits of the tensor-core kernels)
    long long wait_cycles;   // bound of every device-side wait, in SM clock cycles
};

// Launchers (defined in the kernel translation units).  All return the
// cudaError_t of the launch.
cudaError_t launch_simt_scan(const ScanArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_simt_bwd(const BwdArgs &a, bool bf16, cudaStream_t st);
// Tensor-core chunk sums and per-chunk gradients (ssd_bwd_tc.cu): bf16, P = 64, N = 128, one
// group, 128-position chunks (a.Q == 128); launch_simt_bwd uses them in place of its own.
bool bwd_tc_supported(const BwdArgs &a, bool bf16);
cudaError_t launch_bwd_tc_sums(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_bwd_tc_chunk(const BwdArgs &a, cudaStream_t st);

}  // namespace ssd
