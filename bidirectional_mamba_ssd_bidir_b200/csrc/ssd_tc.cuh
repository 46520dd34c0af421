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
    int nseg;                // segments per sequence (1: one CTA walks the whole sequence)
    int npiece;              // pieces each segment's local end state is formed in (nseg > 1)
    bool concurrent;         // run the exact kernel on a side stream beside the shared-score kernel
};

// Scratch of a segmented call, inside the path workspace.
struct SegScratch {
    float *sloc;                        // [batch][H][2][(nseg - 1) npiece][P][N] pieces' local end states
    float *ldec;                        // [batch][H][2][(nseg - 1) npiece] A * (sum of dt per piece), log2
    unsigned long long *steep;          // [batch][H/2][2] epoch-tagged steep-chain marks
};

bool tc_supported(bool bf16, int batch, int L, int H, int P, int N, int G, int chunk);
// Segments per sequence for a call of this shape: enough CTAs to fill the GPU when the
// batch alone does not (at least two blocks per segment).
int tc_segments(int batch, int L, int H);
// Blocks per segment (the last segment may be shorter).
int tc_segment_blocks(int L, int nseg);
// Pieces each of the first nseg - 1 segments is formed in by the segment-state kernel, and
// blocks per piece (a segment's last piece may be shorter).
int tc_state_pieces(int batch, int L, int H, int nseg);
int tc_piece_blocks(int L, int nseg, int npiece);
size_t tc_workspace_bytes(int batch, int L, int H, int chunk, int nseg);
TcArgs make_tc_args(int batch, int L, int H, int chunk, void *ws, int *status);
void tc_set_direction(TcArgs &t, int slot, int dir, const void *x, const void *dt, const float *A,
                      const void *B, const void *C, const float *D);
int tc_launches(bool bidir, int nseg);
cudaError_t launch_tc(const TcArgs &t, bool bidir, void *y, cudaStream_t st);
// the shared-score kernel (ssd_tcs.cu); launch_tc runs it first for calls without a carried state
cudaError_t launch_tcs(const TcArgs &t, bool bidir, void *y, unsigned long long *ticket, unsigned long long *ready,
                       const SegScratch &sc, unsigned long long epoch, cudaStream_t st);
// the segment-state kernel (ssd_tcs_seg.cu): local end states and steep marks, before launch_tcs
cudaError_t launch_segstate(const TcArgs &t, bool bidir, const SegScratch &sc, unsigned long long epoch,
                            cudaStream_t st);
size_t tcs_smem_bytes();

}  // namespace ssd
