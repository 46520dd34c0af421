// Multi-head softmax attention without a mask (the attention mixer of DiffuMamba-H) on the
// tensor core.  See attention.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

struct AttnArgs {
    int batch, L, H, D;                 // D: 64 or 128
    const void *q, *k, *v;              // bf16; token t of sequence b, head h at [(b L + t) ld + h D]
    long long ldq, ldk, ldv;            // elements between consecutive tokens
    void *o;                            // bf16 output, same indexing with ldo
    long long ldo;
    float scale;                        // multiplies q.k before the softmax
    int *status;                        // device status word
    long long wait_cycles;              // bound of every device-side wait
};

bool attention_supported(int D);
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st);

}  // namespace ssd
