// ssd_api.cu -- the C ABI declared in include/bidir_ssd.h: argument checks,
// workspace layout, path choice and stream-ordered launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <string>

#include "../../include/bidir_ssd.h"
#include "attention.cuh"
#include "mixer.cuh"
#include "ssd_internal.cuh"
#include "ssd_tc.cuh"

namespace {

thread_local std::string g_err;

// Process-wide test hooks (ssd_debug_fault): bound of device-side waits and an
// injected fault.  Defaults: 2 s, no fault.
std::atomic<int> g_fault{0};
std::atomic<long long> g_wait_ns{2000000000LL};

// SM clock (kHz) of each device, queried once: converts the wait bound to cycles.
std::atomic<int> g_clock_khz[64];

long long wait_cycles_now() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    int khz = (dev >= 0 && dev < 64) ? g_clock_khz[dev].load(std::memory_order_relaxed) : 0;
    if (khz <= 0) {
        if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0) khz = 2000000;
        if (dev >= 0 && dev < 64) g_clock_khz[dev].store(khz, std::memory_order_relaxed);
    }
    return (long long)((double)g_wait_ns.load() * 1e-9 * (double)khz * 1e3);
}

ssd_status fail(ssd_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

ssd_status cuda_fail(cudaError_t e, const char *what) {
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;   // device status word + padding

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool is_pow2_in(int v, const int *set, int n) {
    for (int i = 0; i < n; ++i)
        if (v == set[i]) return true;
    return false;
}

bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ssd_status check_shape(const ssd_shape *s, int chunk) {
    if (!s) return fail(SSD_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || s->seqlen < 0 || s->nheads <= 0 || s->headdim <= 0 || s->dstate <= 0 || s->ngroups <= 0)
        return fail(SSD_ERR_INVALID_ARG, "negative or zero size in shape");
    if (s->io != SSD_BF16 && s->io != SSD_F32) return fail(SSD_ERR_INVALID_ARG, "unknown io dtype %d", (int)s->io);
    static const int P_ok[] = {16, 32, 64}, N_ok[] = {16, 32, 64, 128}, Q_ok[] = {16, 32, 64, 128, 256};
    if (!is_pow2_in(s->headdim, P_ok, 3)) return fail(SSD_ERR_UNSUPPORTED, "headdim %d not in {16,32,64}", s->headdim);
    if (!is_pow2_in(s->dstate, N_ok, 4)) return fail(SSD_ERR_UNSUPPORTED, "dstate %d not in {16,32,64,128}", s->dstate);
    if (!is_pow2_in(chunk, Q_ok, 5)) return fail(SSD_ERR_UNSUPPORTED, "chunk %d not in {16,32,64,128,256}", chunk);
    if (s->nheads % s->ngroups != 0)
        return fail(SSD_ERR_UNSUPPORTED, "nheads %d not a multiple of ngroups %d", s->nheads, s->ngroups);
    if (s->seqlen % chunk != 0) return fail(SSD_ERR_INVALID_ARG, "seqlen %d not a multiple of chunk %d", s->seqlen, chunk);
    const double elems = (double)s->batch * s->seqlen * s->nheads * s->headdim;
    if (elems > 4.0e9) return fail(SSD_ERR_UNSUPPORTED, "tensor too large (%.3g elements)", elems);
    return SSD_OK;
}

ssd_status check_params(const ssd_params *p, const char *which) {
    if (!p) return fail(SSD_ERR_INVALID_ARG, "%s params is NULL", which);
    if (!aligned16(p->x) || !aligned16(p->B) || !aligned16(p->C))
        return fail(SSD_ERR_INVALID_ARG, "%s: x, B and C must be non-NULL and 16-byte aligned", which);
    if (!p->dt || !p->A) return fail(SSD_ERR_INVALID_ARG, "%s: dt and A must be non-NULL", which);
    if ((reinterpret_cast<uintptr_t>(p->dt) & 3u) || (reinterpret_cast<uintptr_t>(p->A) & 3u) ||
        (reinterpret_cast<uintptr_t>(p->D) & 3u))
        return fail(SSD_ERR_INVALID_ARG, "%s: dt, A, D must be 4-byte aligned", which);
    return SSD_OK;
}

// SIMT-path workspace: [status | decays (batch*H*nc floats) | states (batch*H*nc*P*N floats)].
// A single chunk needs the decays and states only when a state crosses the call boundary
// (ssd_scan_state); the size reported is the larger one.
size_t simt_ws_bytes(const ssd_shape *s, int chunk) {
    const size_t units = (size_t)s->batch * s->nheads * (s->seqlen / chunk);
    return kStatusBytes + round_up(units * sizeof(float)) + round_up(units * s->headdim * s->dstate * sizeof(float));
}

int choose_path(const ssd_shape *s, int chunk) {
    return ssd::tc_supported(s->io == SSD_BF16, s->batch, s->seqlen, s->nheads, s->headdim, s->dstate,
                             s->ngroups, chunk) ? 1 : 0;
}

// Segments per sequence on the tensor-core path (1 when segmenting is not allowed).
int tc_nseg(const ssd_shape *s, bool segments) {
    return segments ? ssd::tc_segments(s->batch, s->seqlen, s->nheads) : 1;
}

size_t path_ws_bytes(const ssd_shape *s, int chunk, bool segments = true) {
    if (choose_path(s, chunk) == 1)
        return kStatusBytes +
               round_up(ssd::tc_workspace_bytes(s->batch, s->seqlen, s->nheads, chunk, tc_nseg(s, segments)));
    return simt_ws_bytes(s, chunk);
}

ssd::ScanArgs make_args(const ssd_shape *s, const ssd_params *p, int dir, int chunk, void *y, void *ws) {
    ssd::ScanArgs a{};
    a.batch = s->batch; a.L = s->seqlen; a.H = s->nheads; a.P = s->headdim; a.N = s->dstate;
    a.G = s->ngroups; a.Q = chunk; a.nc = s->seqlen / chunk; a.dir = dir;
    a.x = p->x; a.dt = p->dt; a.B = p->B; a.C = p->C; a.A = p->A; a.D = p->D;
    a.y = y; a.residual = nullptr; a.gate = 0.f; a.mode = ssd::OUT_WRITE;
    char *w = static_cast<char *>(ws) + kStatusBytes;
    const size_t units = (size_t)s->batch * s->nheads * a.nc;
    a.decays = reinterpret_cast<float *>(w);
    a.states = reinterpret_cast<float *>(w + round_up(units * sizeof(float)));
    a.s_in = nullptr;
    a.s_out = nullptr;
    return a;
}

// Validates the shape and, for a non-empty problem, the output and workspace.
// *empty is set when there is nothing to compute (batch or seqlen zero): the
// call then succeeds without looking at any pointer.
ssd_status common_checks(const ssd_shape *s, int chunk, void *out, void *ws, size_t ws_bytes, bool *empty,
                         bool segments = true) {
    ssd_status st = check_shape(s, chunk);
    if (st != SSD_OK) return st;
    *empty = s->batch == 0 || s->seqlen == 0;
    if (*empty) return SSD_OK;
    if (!aligned16(out)) return fail(SSD_ERR_INVALID_ARG, "output must be non-NULL and 16-byte aligned");
    const size_t need = path_ws_bytes(s, chunk, segments);
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
        return fail(SSD_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    if (ws_bytes < need) return fail(SSD_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
    return SSD_OK;
}

ssd_status run_simt(const ssd_shape *s, const ssd_params *p, int dir, int chunk, void *y, void *ws,
                    int mode, const void *residual, float gate, cudaStream_t st,
                    const float *s_in = nullptr, float *s_out = nullptr) {
    ssd::ScanArgs a = make_args(s, p, dir, chunk, y, ws);
    a.mode = mode; a.residual = residual; a.gate = gate;
    a.s_in = s_in; a.s_out = s_out;
    cudaError_t e = ssd::launch_simt_scan(a, s->io == SSD_BF16, st);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "SIMT scan launch");
}

// The bidirectional mixer.  `fixed_scratch` is the no-allocation entry point: one CTA per
// sequence (its scratch has a fixed size) and every kernel on the caller's stream (no side
// stream is made for it).
ssd_status bidir_run(const ssd_shape *shape, const ssd_params *fwd, const ssd_params *rev, int chunk, void *y,
                     void *workspace, size_t workspace_bytes, void *stream, bool fixed_scratch) {
    const bool segments = !fixed_scratch;
    g_err.clear();
    bool empty = false;
    ssd_status st = common_checks(shape, chunk, y, workspace, workspace_bytes, &empty, segments);
    if (st != SSD_OK || empty) return st;
    if ((st = check_params(fwd, "forward")) != SSD_OK) return st;
    if ((st = check_params(rev, "reverse")) != SSD_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (choose_path(shape, chunk) == 1) {
        ssd::TcArgs t = ssd::make_tc_args(shape->batch, shape->seqlen, shape->nheads, chunk,
                                          static_cast<char *>(workspace) + kStatusBytes,
                                          static_cast<int *>(workspace));
        t.wait_cycles = wait_cycles_now();
        t.fault = g_fault.load();
        t.nseg = tc_nseg(shape, segments);
        t.npiece = ssd::tc_state_pieces(shape->batch, shape->seqlen, shape->nheads, t.nseg);
        t.concurrent = !fixed_scratch;
        ssd::tc_set_direction(t, 0, 1, fwd->x, fwd->dt, fwd->A, fwd->B, fwd->C, fwd->D);
        ssd::tc_set_direction(t, 1, -1, rev->x, rev->dt, rev->A, rev->B, rev->C, rev->D);
        cudaError_t e = ssd::launch_tc(t, /*bidir=*/true, y, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "tensor-core bidirectional launch");
    }
    st = run_simt(shape, fwd, 1, chunk, y, workspace, ssd::OUT_WRITE, nullptr, 0.f, cs);
    if (st != SSD_OK) return st;
    return run_simt(shape, rev, -1, chunk, y, workspace, ssd::OUT_ACCUM, nullptr, 0.f, cs);
}

}  // namespace

extern "C" {

size_t ssd_workspace_bytes(const ssd_shape *shape, int chunk) {
    if (check_shape(shape, chunk) != SSD_OK) return 0;
    return path_ws_bytes(shape, chunk);
}

int ssd_path_for(const ssd_shape *shape, int chunk) {
    if (check_shape(shape, chunk) != SSD_OK) return -1;
    return choose_path(shape, chunk);
}

int ssd_segments_for(const ssd_shape *shape, int chunk) {
    if (check_shape(shape, chunk) != SSD_OK) return -1;
    return choose_path(shape, chunk) == 1 ? tc_nseg(shape, true) : 0;
}

int ssd_kernel_launches(const ssd_shape *shape, int chunk, int op) {
    if (check_shape(shape, chunk) != SSD_OK || op < 0 || op > 2) return -1;
    if (shape->batch == 0 || shape->seqlen == 0) return 0;
    const int dirs = op == 1 ? 2 : 1;
    if (op != 2 && choose_path(shape, chunk) == 1) return ssd::tc_launches(op == 1, tc_nseg(shape, true));
    return dirs * (shape->seqlen / chunk > 1 ? 3 : 1);
}

ssd_status ssd_scan(const ssd_shape *shape, const ssd_params *p, int direction, int chunk, void *y,
                    void *workspace, size_t workspace_bytes, void *stream) {
    g_err.clear();
    bool empty = false;
    ssd_status st = common_checks(shape, chunk, y, workspace, workspace_bytes, &empty);
    if (st != SSD_OK) return st;
    if (direction != 1 && direction != -1) return fail(SSD_ERR_INVALID_ARG, "direction must be +1 or -1");
    if (empty) return SSD_OK;
    if ((st = check_params(p, "scan")) != SSD_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (choose_path(shape, chunk) == 1) {
        ssd::TcArgs t = ssd::make_tc_args(shape->batch, shape->seqlen, shape->nheads, chunk,
                                          static_cast<char *>(workspace) + kStatusBytes,
                                          static_cast<int *>(workspace));
        t.wait_cycles = wait_cycles_now();
        t.fault = g_fault.load();
        ssd::tc_set_direction(t, 0, direction, p->x, p->dt, p->A, p->B, p->C, p->D);
        cudaError_t e = ssd::launch_tc(t, /*bidir=*/false, y, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "tensor-core scan launch");
    }
    return run_simt(shape, p, direction, chunk, y, workspace, ssd::OUT_WRITE, nullptr, 0.f, cs);
}

ssd_status ssd_scan_state(const ssd_shape *shape, const ssd_params *p, int direction, int chunk,
                          const float *state_in, float *state_out, void *y, void *workspace,
                          size_t workspace_bytes, void *stream) {
    g_err.clear();
    ssd_status st = check_shape(shape, chunk);
    if (st != SSD_OK) return st;
    if (direction != 1 && direction != -1) return fail(SSD_ERR_INVALID_ARG, "direction must be +1 or -1");
    if ((reinterpret_cast<uintptr_t>(state_in) & 3u) || (reinterpret_cast<uintptr_t>(state_out) & 3u))
        return fail(SSD_ERR_INVALID_ARG, "states must be 4-byte aligned");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (shape->batch == 0) return SSD_OK;
    if (shape->seqlen == 0) {
        // no token: the state passes through unchanged
        if (!state_out) return SSD_OK;
        const size_t bytes = (size_t)shape->batch * shape->nheads * shape->headdim * shape->dstate * sizeof(float);
        cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, cs)
                                 : cudaMemsetAsync(state_out, 0, bytes, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "state pass-through");
    }
    bool empty = false;
    if ((st = common_checks(shape, chunk, y, workspace, workspace_bytes, &empty)) != SSD_OK) return st;
    if ((st = check_params(p, "scan")) != SSD_OK) return st;
    if (choose_path(shape, chunk) == 1) {
        ssd::TcArgs t = ssd::make_tc_args(shape->batch, shape->seqlen, shape->nheads, chunk,
                                          static_cast<char *>(workspace) + kStatusBytes,
                                          static_cast<int *>(workspace));
        t.wait_cycles = wait_cycles_now();
        t.fault = g_fault.load();
        t.s_in = state_in;
        t.s_out = state_out;
        ssd::tc_set_direction(t, 0, direction, p->x, p->dt, p->A, p->B, p->C, p->D);
        cudaError_t e = ssd::launch_tc(t, /*bidir=*/false, y, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "tensor-core scan launch");
    }
    return run_simt(shape, p, direction, chunk, y, workspace, ssd::OUT_WRITE, nullptr, 0.f, cs, state_in, state_out);
}

size_t ssd_bwd_workspace_bytes(const ssd_shape *shape, int chunk) {
    if (check_shape(shape, chunk) != SSD_OK) return 0;
    const int Q = chunk < 64 ? chunk : 64;
    const size_t nc = (size_t)shape->seqlen / Q, bh = (size_t)shape->batch * shape->nheads;
    const size_t PN = (size_t)shape->headdim * shape->dstate, tokh = (size_t)shape->batch * shape->seqlen * shape->nheads;
    return kStatusBytes + 2 * round_up(bh * nc * PN * sizeof(float)) + 2 * round_up(bh * nc * sizeof(float)) +
           2 * round_up(tokh * shape->dstate * sizeof(float)) + 2 * round_up(tokh * sizeof(float)) +
           2 * round_up(bh * sizeof(float));
}

ssd_status ssd_scan_bwd(const ssd_shape *shape, const ssd_params *p, int direction, int chunk, const void *gy,
                        float *gx, float *gdt, float *gA, float *gB, float *gC, float *gD, void *workspace,
                        size_t workspace_bytes, void *stream) {
    g_err.clear();
    ssd_status st = check_shape(shape, chunk);
    if (st != SSD_OK) return st;
    if (direction != 1 && direction != -1) return fail(SSD_ERR_INVALID_ARG, "direction must be +1 or -1");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (!gA) return fail(SSD_ERR_INVALID_ARG, "gA must be non-NULL");
    const bool empty = shape->batch == 0 || shape->seqlen == 0;
    if (empty) {
        // no token: dA and dD are zero
        cudaError_t e = cudaMemsetAsync(gA, 0, sizeof(float) * shape->nheads, cs);
        if (e == cudaSuccess && gD) e = cudaMemsetAsync(gD, 0, sizeof(float) * shape->nheads, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "empty gradient clear");
    }
    if ((st = check_params(p, "scan")) != SSD_OK) return st;
    if (!aligned16(gy)) return fail(SSD_ERR_INVALID_ARG, "gy must be non-NULL and 16-byte aligned");
    if (!gx || !gdt || !gB || !gC) return fail(SSD_ERR_INVALID_ARG, "gx, gdt, gB and gC must be non-NULL");
    if (!aligned16(gx)) return fail(SSD_ERR_INVALID_ARG, "gx must be 16-byte aligned");
    if (gD && !p->D) return fail(SSD_ERR_INVALID_ARG, "gD requested but D is NULL");
    const size_t need = ssd_bwd_workspace_bytes(shape, chunk);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return fail(SSD_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    if (workspace_bytes < need) return fail(SSD_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
    ssd::BwdArgs a{};
    a.batch = shape->batch; a.L = shape->seqlen; a.H = shape->nheads; a.P = shape->headdim; a.N = shape->dstate;
    // the tensor-core shapes run the gradients in 128-position chunks on tcgen05; others in chunks
    // of at most 64 on the CUDA cores
    const bool tc = choose_path(shape, chunk) == 1;
    a.G = shape->ngroups; a.Q = tc ? 128 : (chunk < 64 ? chunk : 64); a.nc = shape->seqlen / a.Q; a.dir = direction;
    a.status = static_cast<int *>(workspace);
    a.wait_cycles = wait_cycles_now();
    a.x = p->x; a.dt = p->dt; a.B = p->B; a.C = p->C; a.gy = gy; a.A = p->A; a.D = p->D;
    a.gx = gx; a.gdt = gdt; a.gA = gA; a.gB = gB; a.gC = gC; a.gD = gD;
    const size_t nc = a.nc, bh = (size_t)a.batch * a.H, PN = (size_t)a.P * a.N, tokh = (size_t)a.batch * a.L * a.H;
    char *w = static_cast<char *>(workspace) + kStatusBytes;
    auto take = [&](size_t bytes) { float *f = reinterpret_cast<float *>(w); w += round_up(bytes); return f; };
    a.sf = take(bh * nc * PN * sizeof(float));
    a.sg = take(bh * nc * PN * sizeof(float));
    a.dec = take(bh * nc * sizeof(float));
    a.gxd = take(bh * nc * sizeof(float));
    a.gBh = take(tokh * a.N * sizeof(float));
    a.gCh = take(tokh * a.N * sizeof(float));
    a.gcs = take(tokh * sizeof(float));
    a.u = take(tokh * sizeof(float));
    a.gAp = take(bh * sizeof(float));
    a.gDp = take(bh * sizeof(float));
    cudaError_t e = ssd::launch_simt_bwd(a, shape->io == SSD_BF16, cs);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "scan gradient launch");
}

ssd_status bidir_ssd(const ssd_shape *shape, const ssd_params *fwd, const ssd_params *rev, int chunk, void *y,
                     void *workspace, size_t workspace_bytes, void *stream) {
    return bidir_run(shape, fwd, rev, chunk, y, workspace, workspace_bytes, stream, /*fixed_scratch=*/false);
}

ssd_status r2l_block_scan(const ssd_shape *shape, const ssd_params *p, float s, const void *residual, int chunk,
                          void *out, void *workspace, size_t workspace_bytes, void *stream) {
    g_err.clear();
    bool empty = false;
    ssd_status st = common_checks(shape, chunk, out, workspace, workspace_bytes, &empty);
    if (st != SSD_OK || empty) return st;
    if ((st = check_params(p, "r2l")) != SSD_OK) return st;
    if (!aligned16(residual)) return fail(SSD_ERR_INVALID_ARG, "residual must be non-NULL and 16-byte aligned");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (s == 0.0f) {
        // Gate at its initial value: the block is returned untouched, bit for bit.
        if (out == residual) return SSD_OK;
        const size_t bytes = (size_t)shape->batch * shape->seqlen * shape->nheads * shape->headdim *
                             (shape->io == SSD_BF16 ? 2 : 4);
        cudaError_t e = cudaMemcpyAsync(out, residual, bytes, cudaMemcpyDeviceToDevice, cs);
        return e == cudaSuccess ? SSD_OK : cuda_fail(e, "residual copy");
    }
    return run_simt(shape, p, -1, chunk, out, workspace, ssd::OUT_GATE, residual, s, cs);
}

ssd_status ssd_workspace_status(void *workspace, size_t workspace_bytes, void *stream) {
    g_err.clear();
    if (!workspace || workspace_bytes < kStatusBytes) return fail(SSD_ERR_INVALID_ARG, "workspace too small");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (word != 0) {
        e = cudaMemsetAsync(workspace, 0, sizeof(int), cs);
        if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
        if (e != cudaSuccess) return cuda_fail(e, "status clear");
        return fail(SSD_ERR_TIMEOUT, "a bounded device wait gave up (code %d)", word);
    }
    return SSD_OK;
}

const char *ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument";
        case SSD_ERR_UNSUPPORTED: return "unsupported shape";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char *ssd_last_error(void) { return g_err.c_str(); }

ssd_status ssd_debug_fault(int mode, double wait_limit_seconds) {
    g_err.clear();
    if (mode < 0 || mode > 1) return fail(SSD_ERR_INVALID_ARG, "unknown fault mode %d", mode);
    if (!(wait_limit_seconds >= 1e-4 && wait_limit_seconds <= 60.0))
        return fail(SSD_ERR_INVALID_ARG, "wait limit must be within [1e-4, 60] seconds");
    g_fault.store(mode);
    g_wait_ns.store((long long)(wait_limit_seconds * 1e9));
    return SSD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// bidir_ssd_noalloc: the bidirectional mixer with its scratch in a fixed
// device array of this library instead of a caller-supplied workspace.

namespace {

// The scratch: status area first, then what the chosen path keeps between the
// kernels (hand-off flags on the tensor-core path, chunk decays and states on
// the SIMT path).  Zero at module load; the parts that must start at zero are
// cleared again at every call.
__device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_MAX_SCRATCH_BYTES];

// Its device address in the current device's context.  Looked up on every call
// (cudaGetSymbolAddress allocates nothing): a cached address would go stale if
// the context were destroyed (cudaDeviceReset) and the library's module loaded
// again at another address, or if the caller switched to another context on the
// same device.  A host-side reference to the array itself is never a device address.
ssd_status noalloc_scratch(void **out) {
    void *ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the scratch array");
    if (!ptr) return fail(SSD_ERR_CUDA, "cudaGetSymbolAddress returned NULL");
    *out = ptr;
    return SSD_OK;
}

}  // namespace

extern "C" {

ssd_status bidir_ssd_noalloc(const ssd_shape *shape, const ssd_params *fwd, const ssd_params *rev, int chunk,
                             void *y, void *stream, void **status_area) {
    g_err.clear();
    if (status_area) *status_area = nullptr;
    ssd_status st = check_shape(shape, chunk);
    if (st != SSD_OK) return st;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    const size_t need = path_ws_bytes(shape, chunk, /*segments=*/false);
    if (need > (size_t)SSD_NOALLOC_MAX_SCRATCH_BYTES)
        return fail(SSD_ERR_UNSUPPORTED,
                    "this shape needs %zu bytes of scratch, more than the %zu the no-allocation entry point "
                    "holds; call bidir_ssd with a workspace instead",
                    need, (size_t)SSD_NOALLOC_MAX_SCRATCH_BYTES);
    void *ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != SSD_OK) return st;
    // the status word, and on the tensor-core path the hand-off flags, start at zero
    const size_t clear = choose_path(shape, chunk) == 1 ? need : kStatusBytes;
    cudaError_t e = cudaMemsetAsync(ws, 0, clear, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "scratch clear");
    st = bidir_run(shape, fwd, rev, chunk, y, ws, (size_t)SSD_NOALLOC_MAX_SCRATCH_BYTES, stream, /*fixed_scratch=*/true);
    if (st == SSD_OK && status_area) *status_area = ws;
    return st;
}

}  // extern "C"

// ---------------------------------------------------------------- the mixer around the scan

namespace {

struct MixerLayout {
    int chunk;
    ssd_shape scan;
    size_t scan_ws, zx, x, b, c, dt, y, ynf, ynr, total;
};

ssd_status mixer_layout(const ssd_mixer_shape *s, MixerLayout *lo) {
    if (!s) return fail(SSD_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || s->seqlen < 0 || s->d_model <= 0 || s->nheads <= 0)
        return fail(SSD_ERR_INVALID_ARG, "negative or zero size in mixer shape");
    if (s->headdim != 64 || s->dstate != 128 || s->ngroups != 1 || s->nheads % 8 != 0)
        return fail(SSD_ERR_UNSUPPORTED, "mixer needs headdim 64, dstate 128, one group, heads a multiple of 8");
    if (s->d_model % 64 != 0 || s->seqlen % 128 != 0 || s->d_conv < 1 || s->d_conv > 8)
        return fail(SSD_ERR_UNSUPPORTED, "mixer needs d_model %% 64 == 0, seqlen %% 128 == 0, d_conv in 1..8");
    if (s->nheads > 256) return fail(SSD_ERR_UNSUPPORTED, "mixer takes at most 256 heads (d_inner 16384)");
    const int di = s->nheads * s->headdim;   // a multiple of 512
    lo->chunk = s->seqlen % 256 == 0 ? 256 : 128;
    lo->scan = ssd_shape{s->batch, s->seqlen, s->nheads, s->headdim, s->dstate, s->ngroups, SSD_BF16};
    const size_t M = (size_t)s->batch * s->seqlen, N = (size_t)s->ngroups * s->dstate;
    const size_t dinp = 2 * (size_t)di + 2 * N + s->nheads;
    lo->scan_ws = round_up(path_ws_bytes(&lo->scan, lo->chunk));
    size_t o = lo->scan_ws;
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    lo->zx = take(M * dinp * 2);
    lo->x = take(M * di * 2);
    lo->b = take(M * N * 2);
    lo->c = take(M * N * 2);
    lo->dt = take(M * s->nheads * 2);
    lo->y = take(M * di * 2);
    lo->ynf = take(M * di * 2);
    lo->ynr = take(M * di * 2);
    lo->total = o;
    return SSD_OK;
}

}  // namespace

extern "C" {

size_t ssd_mixer_workspace_bytes(const ssd_mixer_shape *shape) {
    MixerLayout lo;
    return mixer_layout(shape, &lo) == SSD_OK ? lo.total : 0;
}

ssd_status ssd_gemm_bf16(int M, int N, int K, const void *A, const void *W, void *D, void *workspace,
                         size_t workspace_bytes, void *stream) {
    g_err.clear();
    if (M < 0 || N < 0 || K < 0) return fail(SSD_ERR_INVALID_ARG, "negative GEMM size");
    if (M == 0 || N == 0) return SSD_OK;
    if (!ssd::mixer_gemm_supported(M, N, K))
        return fail(SSD_ERR_UNSUPPORTED, "GEMM needs M %% 128 == 0, K %% 64 == 0, N %% 8 == 0 (and the TMA encoder)");
    if (!aligned16(A) || !aligned16(W) || !aligned16(D)) return fail(SSD_ERR_INVALID_ARG, "A, W, D must be 16-byte aligned");
    if (!workspace || workspace_bytes < kStatusBytes) return fail(SSD_ERR_INVALID_ARG, "workspace of 256 bytes needed");
    ssd::GemmArgs g{};
    g.M = M; g.N = N; g.k1 = K; g.k2 = 0; g.A1 = A; g.W1 = W; g.D = D;
    g.status = static_cast<int *>(workspace);
    g.wait_cycles = wait_cycles_now();
    cudaError_t e = ssd::launch_gemm_bf16(g, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "GEMM launch");
}

ssd_status mamba2_mixer_bidir(const ssd_mixer_shape *shape, const void *u, const ssd_mixer_layer *fwd,
                              const ssd_mixer_layer *rev, void *out, void *workspace, size_t workspace_bytes,
                              void *stream) {
    g_err.clear();
    MixerLayout lo;
    ssd_status st = mixer_layout(shape, &lo);
    if (st != SSD_OK) return st;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    if (!aligned16(u) || !aligned16(out)) return fail(SSD_ERR_INVALID_ARG, "u and out must be 16-byte aligned");
    if (!fwd || !rev) return fail(SSD_ERR_INVALID_ARG, "layer weights are NULL");
    for (const ssd_mixer_layer *l : {fwd, rev})
        if (!aligned16(l->W_in) || !aligned16(l->W_out) || !l->conv_w || !l->conv_b || !l->dt_bias || !l->A || !l->D ||
            !aligned16(l->norm_w))
            return fail(SSD_ERR_INVALID_ARG, "a layer weight is NULL (or W_in, W_out, norm_w not 16-byte aligned)");
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return fail(SSD_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    if (workspace_bytes < lo.total) return fail(SSD_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, lo.total);
    if (!ssd::mixer_gemm_supported(shape->batch * shape->seqlen, 8, shape->d_model))
        return fail(SSD_ERR_UNSUPPORTED, "tensor-core GEMM unavailable for this shape");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    const int M = shape->batch * shape->seqlen, di = shape->nheads * shape->headdim, N = shape->dstate;
    const int cd = di + 2 * N, dinp = 2 * di + 2 * N + shape->nheads;
    auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16 *>(ws + off); };
    int *status = static_cast<int *>(workspace);   // the scan's status word: one for the whole call
    const long long wc = wait_cycles_now();
    cudaError_t e;
    for (int li = 0; li < 2; ++li) {
        const ssd_mixer_layer *L_ = li ? rev : fwd;
        ssd::GemmArgs g{};
        g.M = M; g.N = dinp; g.k1 = shape->d_model; g.k2 = 0; g.A1 = u; g.W1 = L_->W_in; g.D = bf(lo.zx);
        g.status = status; g.wait_cycles = wc;
        if ((e = ssd::launch_gemm_bf16(g, cs)) != cudaSuccess) return cuda_fail(e, "input projection");
        ssd::MixerConvArgs ca{};
        ca.batch = shape->batch; ca.L = shape->seqlen; ca.d_inner = di; ca.N = N; ca.H = shape->nheads;
        ca.conv_dim = cd; ca.d_in_proj = dinp; ca.K = shape->d_conv; ca.dir = li ? -1 : 1;
        ca.zxbcdt = bf(lo.zx); ca.conv_w = L_->conv_w; ca.conv_b = L_->conv_b; ca.dt_bias = L_->dt_bias;
        ca.x = bf(lo.x); ca.B = bf(lo.b); ca.C = bf(lo.c); ca.dt = bf(lo.dt);
        if ((e = ssd::launch_conv_silu_dt(ca, cs)) != cudaSuccess) return cuda_fail(e, "convolution");
        const ssd_params p{bf(lo.x), bf(lo.dt), L_->A, bf(lo.b), bf(lo.c), L_->D};
        if ((st = ssd_scan(&lo.scan, &p, li ? -1 : 1, lo.chunk, bf(lo.y), workspace, lo.scan_ws, stream)) != SSD_OK)
            return st;
        ssd::MixerNormArgs na{};
        na.batch = shape->batch; na.L = shape->seqlen; na.d_inner = di; na.d_in_proj = dinp; na.eps = 1e-5f;
        na.y = bf(lo.y); na.zxbcdt = bf(lo.zx); na.w = L_->norm_w; na.out = bf(li ? lo.ynr : lo.ynf);
        if ((e = ssd::launch_gated_norm(na, cs)) != cudaSuccess) return cuda_fail(e, "gated norm");
    }
    ssd::GemmArgs g{};
    g.M = M; g.N = shape->d_model; g.k1 = di; g.k2 = di;
    g.A1 = bf(lo.ynf); g.W1 = fwd->W_out; g.A2 = bf(lo.ynr); g.W2 = rev->W_out; g.D = out;
    g.status = status; g.wait_cycles = wc;
    if ((e = ssd::launch_gemm_bf16(g, cs)) != cudaSuccess) return cuda_fail(e, "output projection");
    g_err.clear();
    return SSD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- the DiffuMamba-H attention mixer

namespace {

ssd_status attn_checks(const ssd_attn_shape *s) {
    if (!s) return fail(SSD_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0 || s->seqlen < 0 || s->nheads <= 0 || s->headdim <= 0)
        return fail(SSD_ERR_INVALID_ARG, "negative or zero size in attention shape");
    if (s->batch > 65535 || s->nheads > 65535) return fail(SSD_ERR_UNSUPPORTED, "batch and heads up to 65535");
    if (!ssd::attention_supported(s->headdim))
        return fail(SSD_ERR_UNSUPPORTED, "attention needs headdim 64 or 128 (and the TMA encoder)");
    return SSD_OK;
}

ssd_status attn_run(const ssd_attn_shape *s, const void *q, long long ldq, const void *k, long long ldk,
                    const void *v, long long ldv, void *out, long long ldo, float scale, int *status,
                    cudaStream_t cs) {
    const long long w = (long long)s->nheads * s->headdim;
    for (long long ld : {ldq, ldk, ldv, ldo})
        if (ld < w || ld % 8 != 0) return fail(SSD_ERR_INVALID_ARG, "row strides must be >= nheads*headdim and multiples of 8");
    ssd::AttnArgs a{};
    a.batch = s->batch; a.L = s->seqlen; a.H = s->nheads; a.D = s->headdim;
    a.q = q; a.k = k; a.v = v; a.o = out;
    a.ldq = ldq; a.ldk = ldk; a.ldv = ldv; a.ldo = ldo;
    a.scale = scale != 0.f ? scale : 1.f / sqrtf((float)s->headdim);
    a.status = status;
    a.wait_cycles = wait_cycles_now();
    cudaError_t e = ssd::launch_attention(a, cs);
    return e == cudaSuccess ? SSD_OK : cuda_fail(e, "attention launch");
}

}  // namespace

extern "C" {

ssd_status ssd_attention(const ssd_attn_shape *shape, const void *q, long long ldq, const void *k, long long ldk,
                         const void *v, long long ldv, void *out, long long ldo, float scale, void *workspace,
                         size_t workspace_bytes, void *stream) {
    g_err.clear();
    ssd_status st = attn_checks(shape);
    if (st != SSD_OK) return st;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(SSD_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
    if (!workspace || workspace_bytes < kStatusBytes) return fail(SSD_ERR_INVALID_ARG, "workspace of 256 bytes needed");
    return attn_run(shape, q, ldq, k, ldk, v, ldv, out, ldo, scale, static_cast<int *>(workspace),
                    static_cast<cudaStream_t>(stream));
}

size_t ssd_attention_block_workspace_bytes(const ssd_attn_shape *shape) {
    if (attn_checks(shape) != SSD_OK) return 0;
    const size_t M = (size_t)shape->batch * shape->seqlen, w = (size_t)shape->nheads * shape->headdim;
    return kStatusBytes + round_up(M * 3 * w * 2) + round_up(M * w * 2);
}

ssd_status attention_block(const ssd_attn_shape *shape, int d_model, const void *u, const void *W_qkv,
                           const void *W_o, void *out, void *workspace, size_t workspace_bytes, void *stream) {
    g_err.clear();
    ssd_status st = attn_checks(shape);
    if (st != SSD_OK) return st;
    if (shape->batch == 0 || shape->seqlen == 0) return SSD_OK;
    const int M = shape->batch * shape->seqlen, w = shape->nheads * shape->headdim;
    if (d_model <= 0 || d_model % 64 != 0 || M % 128 != 0)
        return fail(SSD_ERR_UNSUPPORTED, "attention block needs d_model %% 64 == 0 and batch*seqlen %% 128 == 0");
    if (!ssd::mixer_gemm_supported(M, 3 * w, d_model) || !ssd::mixer_gemm_supported(M, d_model, w))
        return fail(SSD_ERR_UNSUPPORTED, "tensor-core GEMM unavailable for this shape");
    if (!aligned16(u) || !aligned16(W_qkv) || !aligned16(W_o) || !aligned16(out))
        return fail(SSD_ERR_INVALID_ARG, "u, W_qkv, W_o and out must be 16-byte aligned");
    const size_t need = ssd_attention_block_workspace_bytes(shape);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)))
        return fail(SSD_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    if (workspace_bytes < need) return fail(SSD_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    int *status = static_cast<int *>(workspace);
    __nv_bfloat16 *qkv = reinterpret_cast<__nv_bfloat16 *>(ws + kStatusBytes);
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(ws + kStatusBytes + round_up((size_t)M * 3 * w * 2));
    const long long wc = wait_cycles_now();
    cudaError_t e;
    ssd::GemmArgs g{};
    g.M = M; g.N = 3 * w; g.k1 = d_model; g.A1 = u; g.W1 = W_qkv; g.D = qkv;
    g.status = status; g.wait_cycles = wc;
    if ((e = ssd::launch_gemm_bf16(g, cs)) != cudaSuccess) return cuda_fail(e, "q/k/v projection");
    // q, k, v: column blocks of the projection, 3 w elements between tokens
    if ((st = attn_run(shape, qkv, 3LL * w, qkv + w, 3LL * w, qkv + 2 * w, 3LL * w, o, w, 0.f, status, cs)) != SSD_OK)
        return st;
    ssd::GemmArgs g2{};
    g2.M = M; g2.N = d_model; g2.k1 = w; g2.A1 = o; g2.W1 = W_o; g2.D = out;
    g2.status = status; g2.wait_cycles = wc;
    if ((e = ssd::launch_gemm_bf16(g2, cs)) != cudaSuccess) return cuda_fail(e, "output projection");
    g_err.clear();
    return SSD_OK;
}

}  // extern "C"
