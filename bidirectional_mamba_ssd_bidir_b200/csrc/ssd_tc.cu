// ssd_tc.cu -- tensor-core path (not yet enabled).
#include "ssd_tc.cuh"

namespace ssd {

bool tc_supported(bool, int, int, int, int, int, int, int) { return false; }
size_t tc_workspace_bytes(int, int, int, int) { return 0; }
TcArgs make_tc_args(int batch, int L, int H, int chunk, void *ws, int *status) {
    TcArgs t{};
    t.batch = batch; t.L = L; t.H = H; t.chunk = chunk; t.ws = ws; t.status = status;
    return t;
}
void tc_set_direction(TcArgs &t, int slot, int dir, const void *x, const void *dt, const float *A,
                      const void *B, const void *C, const float *D) {
    t.d[slot] = TcDir{x, dt, B, C, A, D, dir};
}
int tc_launches(bool) { return 1; }
cudaError_t launch_tc(const TcArgs &, bool, void *, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace ssd
