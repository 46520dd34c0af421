// ssd_tc.cuh -- launch interface of the tensor-core (tcgen05) path.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ssd {

struct TcDir {
    const void *x, *dt, *B, *C;
    const float *A, *D;
    int dir;
};

struct TcArgs {
    int batch, L, H, chunk;
    TcDir d[2];
    void *ws;          // path scratch (after the status word)
    int *status;       // device status word
    long long wait_cycles;   // bound of every device-side wait, in SM clock cycles
    int fault;               // test hook (0 = none)
    const float *s_in;       // single direction only: [batch][H][P][N] state entering the scan, or null
    float *s_out;            // single direction only: [batch][H][P][N] state leaving the scan, or null
};

bool tc_supported(bool bf16, int batch, int L, int H, int P, int N, int G, int chunk);
size_t tc_workspace_bytes(int batch, int L, int H, int chunk);
TcArgs make_tc_args(int batch, int L, int H, int chunk, void *ws, int *status);
void tc_set_direction(TcArgs &t, int slot, int dir, const void *x, const void *dt, const float *A,
                      const void *B, const void *C, const float *D);
int tc_launches(bool bidir);
cudaError_t launch_tc(const TcArgs &t, bool bidir, void *y, cudaStream_t st);
// the shared-score kernel (ssd_tcs.cu); launch_tc runs it first for calls without a carried state
cudaError_t launch_tcs(const TcArgs &t, bool bidir, void *y, unsigned long long *ticket, unsigned long long *ready,
                       unsigned long long *deferred, unsigned long long epoch, cudaStream_t st);
size_t tcs_smem_bytes();

}  // namespace ssd
