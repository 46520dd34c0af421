// mixer.cuh -- launch interface of the Mamba-2 block's kernels around the scan (mixer.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ssd {

// D[M][N] = A1[M][k1] W1[N][k1]^T (+ A2[M][k2] W2[N][k2]^T when k2 > 0); bf16 in and out,
// float32 accumulation.  M a multiple of 128, k1, k2 multiples of 64, N a multiple of 8.
struct GemmArgs {
    int M, N, k1, k2;
    const void *A1, *W1, *A2, *W2;
    void *D;
    int *status;
    long long wait_cycles;
};
bool mixer_gemm_supported(int M, int N, int K);
cudaError_t launch_gemm_bf16(const GemmArgs &g, cudaStream_t st);

// zxbcdt [batch*L][d_in_proj] -> x [..][d_inner], B, C [..][N], dt [..][H] (bf16): depthwise
// convolution of width K over the sequence (dir > 0: earlier tokens, dir < 0: later ones) with
// bias, then SiLU; dt = softplus(dt_raw + dt_bias).
struct MixerConvArgs {
    int batch, L, d_inner, N, H, conv_dim, d_in_proj, K, dir;
    const __nv_bfloat16 *zxbcdt;
    const float *conv_w, *conv_b, *dt_bias;
    __nv_bfloat16 *x, *B, *C, *dt;
};
cudaError_t launch_conv_silu_dt(const MixerConvArgs &a, cudaStream_t st);

// out = (y * silu(z)) / sqrt(mean over d_inner + eps) * w, z = zxbcdt[..][0:d_inner]
struct MixerNormArgs {
    int batch, L, d_inner, d_in_proj;
    float eps;
    const __nv_bfloat16 *y, *zxbcdt;
    const float *w;
    __nv_bfloat16 *out;
};
cudaError_t launch_gated_norm(const MixerNormArgs &a, cudaStream_t st);

}  // namespace ssd
