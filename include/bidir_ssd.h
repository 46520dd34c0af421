/*
 * bidir_ssd.h -- C ABI of the bidirectional selective state-space (SSD) scan
 * library for NVIDIA B200 (sm_100a).
 *
 * The operation.  Per batch b and head h (group g = h / (nheads/ngroups)),
 * with a state S in R^{headdim x dstate} that starts at zero, the scan visits
 * the tokens in order and computes
 *
 *     S   <- exp(dt[b,t,h] * A[h]) * S + dt[b,t,h] * x[b,t,h,:] (outer) B[b,t,g,:]
 *     y[b,t,h,p] = sum_n C[b,t,g,n] * S[p,n] + D[h] * x[b,t,h,p]
 *
 * This is the Mamba-2 selective scan named by "DiffuMamba: High-Throughput
 * Diffusion LMs with Mamba Backbone" (technical summary, section 2
 * Methodology: the attention mixer is replaced by bidirectional Mamba-2
 * layers) and by "Bifocal Diffusion Language Models" (section 2, mechanism:
 * the right-to-left stream flips the sequence, applies the selective scan and
 * flips back).  The pages do not print the recurrence; the standard Mamba-2
 * form with one scalar decay per head is the one implemented.
 *
 * Layouts.  Every tensor is row-major and contiguous:
 *     x, y      [batch][seqlen][nheads][headdim]      (io dtype)
 *     dt        [batch][seqlen][nheads]               (io dtype, already positive)
 *     B, C      [batch][seqlen][ngroups][dstate]      (io dtype)
 *     A, D      [nheads]                              (float32 always; D may be NULL = no skip term)
 *     residual, out  [batch][seqlen][nheads*headdim]  (io dtype)
 * Arithmetic is float32 (the state is float32) for both io dtypes; bf16
 * outputs are rounded to nearest even once at the end.
 *
 * Ownership.  The caller allocates every buffer; all data pointers are DEVICE
 * pointers on the current CUDA device.  The library allocates nothing on any
 * call below.  Calls are asynchronous and ordered on `stream` (a
 * cudaStream_t passed as void*; NULL = the legacy default stream).  `y` must
 * not overlap any input.  `out` may be the same buffer as `residual`.
 * Data pointers must be 16-byte aligned.
 *
 * Workspace.  Some paths keep scratch data in global memory (chunk states,
 * direction hand-off flags, the device status word).  Query its size with
 * ssd_workspace_bytes() for the exact shape and chunk and pass a device
 * buffer of at least that size.  Its first 256 bytes hold the status word:
 * they must be zero before the workspace's first use.  Calls write them only
 * to record a device-side timeout, and ssd_workspace_status() clears them.
 * The rest needs no initialisation and is not meaningful after the call.
 * Calls that share a workspace must not run concurrently.
 *
 * Errors.  Every entry point returns an ssd_status; no exception or abort
 * crosses the ABI.  Arguments are checked on the host before anything is
 * launched: SSD_ERR_INVALID_ARG for NULL/misaligned pointers, negative sizes,
 * seqlen % chunk != 0 or a short workspace; SSD_ERR_UNSUPPORTED for sizes
 * outside the supported set (headdim in {16,32,64}, dstate in {16,32,64,128},
 * chunk in {16,32,64,128,256}, nheads % ngroups == 0).  A launch failure
 * returns SSD_ERR_CUDA.  Device-side waits are bounded: a wait that gives up
 * records SSD_ERR_TIMEOUT in the workspace status word, which
 * ssd_workspace_status() reports.  ssd_last_error() gives a text for the most
 * recent failure on the calling thread.  There is no CPU fallback: a shape
 * the GPU kernels do not cover is refused.
 */
#ifndef BIDIR_SSD_H
#define BIDIR_SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,
    SSD_ERR_UNSUPPORTED = 2,
    SSD_ERR_CUDA = 3,
    SSD_ERR_TIMEOUT = 4
} ssd_status;

typedef enum { SSD_BF16 = 0, SSD_F32 = 1 } ssd_dtype;

typedef struct {
    int batch, seqlen, nheads, headdim, dstate, ngroups;
    ssd_dtype io;             /* dtype of x, dt, B, C, y, residual, out */
} ssd_shape;

typedef struct {
    const void *x;            /* [batch][seqlen][nheads][headdim] */
    const void *dt;           /* [batch][seqlen][nheads], positive */
    const float *A;           /* [nheads], the per-head decay rate (negative) */
    const void *B;            /* [batch][seqlen][ngroups][dstate] */
    const void *C;            /* [batch][seqlen][ngroups][dstate] */
    const float *D;           /* [nheads] or NULL */
} ssd_params;

/* Bytes of device workspace that ssd_scan, bidir_ssd and r2l_block_scan need
 * for this shape and chunk (the largest of the three).  Returns 0 for shapes
 * the library refuses (the call itself then reports why). */
size_t ssd_workspace_bytes(const ssd_shape *shape, int chunk);

/* One direction of the scan.  direction = +1 visits t = 0..L-1; direction = -1
 * visits t = L-1..0, i.e. y = flip(scan(flip(x, dt, B, C))) with the flip done
 * in the address arithmetic ("Bifocal Diffusion Language Models", section 2,
 * mechanism).  `chunk` is the length of the blocks of the chunked
 * (state-passing) evaluation; the result is the same for every chunk up to
 * float32 rounding.  Writes y. */
ssd_status ssd_scan(const ssd_shape *shape, const ssd_params *p, int direction, int chunk,
                    void *y, void *workspace, size_t workspace_bytes, void *stream);

/* ssd_scan with the state carried across the call boundary, for block-wise
 * decoding: the DiffuMamba page (technical summary, section 2, training and
 * inference: block diffusion with cache reuse; section 4, block caching)
 * reuses what precedes a block, and for a Mamba layer that is this state.
 *
 * state_in  [batch][nheads][headdim][dstate] float32: the state S before the
 *           first token in scan order (the token at t = 0 forward, t = L-1
 *           reverse); NULL = zero, which makes the call ssd_scan.
 * state_out [batch][nheads][headdim][dstate] float32: receives S after the
 *           last token in scan order; NULL = not wanted.
 * Both are device pointers, 4-byte aligned; state_in and state_out may be the
 * same buffer.  Scanning a sequence in pieces, each piece starting from the
 * previous piece's state_out, gives the y and final state of the whole
 * sequence up to rounding.  seqlen = 0 copies state_in to state_out (or zeroes
 * it).  Same layouts, workspace and errors as ssd_scan. */
ssd_status ssd_scan_state(const ssd_shape *shape, const ssd_params *p, int direction, int chunk,
                          const float *state_in, float *state_out, void *y,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Gradients of ssd_scan (zero starting state), for training the layers that
 * run it (the DiffuMamba page, technical summary, section 2, trains the Mamba
 * backbone).  Given gy = dL/dy ([batch][seqlen][nheads][headdim], io dtype)
 * it writes, all float32 device arrays:
 *     gx  [batch][seqlen][nheads][headdim]      dL/dx
 *     gdt [batch][seqlen][nheads]               dL/ddt
 *     gA  [nheads]                              dL/dA, summed over the batch
 *     gB  [batch][seqlen][ngroups][dstate]      dL/dB, summed over the heads of a group
 *     gC  [batch][seqlen][ngroups][dstate]      dL/dC, likewise
 *     gD  [nheads] or NULL                      dL/dD (NULL when p->D is NULL)
 * The bidirectional mixer's gradients are the two directions' gradients for
 * the same gy (y is their sum).  Runs on the CUDA cores in float32, chunked
 * like the forward scan (at most 64 positions per chunk).  gy and gx must be
 * 16-byte aligned; workspace must be 256-byte aligned and hold
 * ssd_bwd_workspace_bytes(shape, chunk) bytes.  Errors as for ssd_scan. */
size_t ssd_bwd_workspace_bytes(const ssd_shape *shape, int chunk);
ssd_status ssd_scan_bwd(const ssd_shape *shape, const ssd_params *p, int direction, int chunk,
                        const void *gy, float *gx, float *gdt, float *gA, float *gB, float *gC,
                        float *gD, void *workspace, size_t workspace_bytes, void *stream);

/* The DiffuMamba bidirectional mixer ("DiffuMamba", technical summary,
 * section 2: a forward and a reverse Mamba layer, independent of each other,
 * for a symmetric context): y = scan(fwd, +1) + scan(rev, -1), the two
 * directions with their own parameter sets (pass the same pointers twice to
 * share them).  Writes y. */
ssd_status bidir_ssd(const ssd_shape *shape, const ssd_params *fwd, const ssd_params *rev,
                     int chunk, void *y, void *workspace, size_t workspace_bytes, void *stream);

/* The R2LM right-to-left sidecar over one generation block ("Bifocal
 * Diffusion Language Models", section 2: the reverse scan's output is a
 * residual correction scaled by the learnable scalar s, initialised to 0 so
 * the model starts bit-identical to its causal baseline; at decode time only
 * the generation block is scanned, with nothing entering from the right):
 *     out = residual + s * scan(p, -1)   for s != 0
 *     out = residual (bit for bit)        for s == 0
 * residual/out are [batch][seqlen][nheads*headdim]. */
ssd_status r2l_block_scan(const ssd_shape *shape, const ssd_params *p, float s,
                          const void *residual, int chunk, void *out,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Largest scratch, in bytes, that bidir_ssd_noalloc holds (status area plus
 * what the chosen path needs; ssd_workspace_bytes gives that figure). */
#define SSD_NOALLOC_MAX_SCRATCH_BYTES (2u << 20)

/* bidir_ssd without a workspace argument.  The pages have no counterpart: it
 * is a convenience of this library for callers that cannot allocate device
 * memory at the point of the call -- a host program whose device memory is
 * all handed out up front (a serving engine's fixed pool), or a latency-bound
 * loop that cannot afford cudaMalloc/cudaFree, which may synchronise the whole
 * device.  The scratch is a fixed 2 MiB array inside this library (one per
 * device); nothing is allocated, by this call or by the library.
 *
 * Same operation, arguments, layouts and results as bidir_ssd.  Shapes whose
 * scratch (ssd_workspace_bytes) exceeds SSD_NOALLOC_MAX_SCRATCH_BYTES are
 * refused with SSD_ERR_UNSUPPORTED before anything is launched; use
 * bidir_ssd with a workspace for them.  Each call first clears, on `stream`,
 * the part of the scratch that must start at zero (the status word and the
 * forward/reverse hand-off flags).
 *
 * Every call looks up the array's address in the current device's context
 * (cudaGetSymbolAddress, which allocates nothing), so it stays right after a
 * cudaDeviceReset or in another context.  The first call on a device also
 * makes the CUDA runtime load this library's kernels there: make that first
 * call before any stream capture.  All calls on one device share the one array: two calls whose
 * work overlaps on the GPU (different streams, no ordering between them) race
 * on it and give wrong results.  Order them on one stream, or with events.
 *
 * status_area (may be NULL) receives the device address of the scratch's
 * 256-byte status area; pass it to ssd_workspace_status(area, 256, stream)
 * to learn whether a bounded device-side wait gave up.  The next call clears
 * it. */
ssd_status bidir_ssd_noalloc(const ssd_shape *shape, const ssd_params *fwd, const ssd_params *rev,
                             int chunk, void *y, void *stream, void **status_area);

/* Waits for `stream`, then reads and clears the device status word in
 * `workspace` (SSD_OK, or SSD_ERR_TIMEOUT if a bounded device-side wait gave
 * up during an earlier call that used this workspace). */
ssd_status ssd_workspace_status(void *workspace, size_t workspace_bytes, void *stream);

/* Static text for a status code. */
const char *ssd_status_string(ssd_status s);

/* Text describing the most recent failure on the calling thread ("" if none). */
const char *ssd_last_error(void);

/* Number of kernels one call launches for this shape and chunk; op: 0 =
 * ssd_scan, 1 = bidir_ssd, 2 = r2l_block_scan with s != 0.  -1 if refused. */
int ssd_kernel_launches(const ssd_shape *shape, int chunk, int op);

/* Test hook for failure detection (process-wide; not for production use).
 * Sets the bound of every device-side wait (default 2 s) and an injected
 * fault: mode 0 = none; mode 1 = in the tensor-core bidirectional mixer the
 * direction that finishes a block first never publishes its part, so the
 * other direction's bounded wait runs out and the call records
 * SSD_ERR_TIMEOUT in the workspace status word (read it with
 * ssd_workspace_status).  No GPU fault, trap or hang is involved: the waiting
 * CTA gives up, drains its copies and exits.  Returns SSD_ERR_INVALID_ARG for
 * an unknown mode or a limit outside [1e-4, 60] s. */
ssd_status ssd_debug_fault(int mode, double wait_limit_seconds);

/* Which kernel family a call with this shape and chunk runs:
 * 1 = tensor-core (tcgen05) path, 0 = SIMT path, -1 = refused. */
int ssd_path_for(const ssd_shape *shape, int chunk);

/* Segments each sequence is cut into on the tensor-core path (SSD / Mamba-2
 * state passing, "DiffuMamba" technical summary section 2: the scan is linear
 * in its state, so a sequence split into runs of whole 128-token blocks is
 * scanned run by run in parallel from the states the runs before it leave).
 * A call cuts its sequences when batch x heads gives fewer CTAs than the GPU
 * has SMs: a first kernel forms each segment's local end state, the scan then
 * runs every segment from the state folded from those before it.  1 = one CTA
 * walks each whole sequence; 0 on the SIMT path; -1 if the shape is refused.
 * bidir_ssd_noalloc never segments. */
int ssd_segments_for(const ssd_shape *shape, int chunk);

/* ------------------------------------------------------------------------
 * The Mamba-2 mixer around the scan.
 *
 * "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", technical
 * summary section 2: the mixer is two independent Mamba-2 layers, one run
 * forward and one on the reversed sequence, summed.  The page does not spell
 * out a layer; it is read as the standard Mamba-2 block:
 *
 *   zxbcdt = u W_in^T                      (no bias; z | xBC | dt_raw)
 *   xBC    = silu(conv(xBC) + conv_b)      (depthwise, width d_conv, causal in the layer's order)
 *   dt     = softplus(dt_raw + dt_bias)
 *   y      = ssd_scan(x, dt, A, B, C, D)   (x, B, C split from xBC)
 *   out    = (rmsnorm(y * silu(z)) * norm_w) W_out^T     (mean over d_inner, eps 1e-5)
 *
 * and the mixer output is layer_fwd(u) + flip(layer_rev(flip(u))).
 * ------------------------------------------------------------------------ */
typedef struct {
    int batch, seqlen;       /* tokens: batch x seqlen, seqlen a multiple of 128 */
    int d_model;             /* a multiple of 64 */
    int nheads, headdim, dstate, ngroups;   /* headdim 64, dstate 128, ngroups 1, nheads % 8 == 0, <= 256 */
    int d_conv;              /* 1 .. 8 */
} ssd_mixer_shape;

/* One layer's weights; device pointers, row-major.  d_inner = nheads * headdim,
 * conv_dim = d_inner + 2 ngroups dstate, d_in_proj = 2 d_inner + 2 ngroups dstate + nheads. */
typedef struct {
    const void *W_in;        /* bf16 [d_in_proj][d_model] */
    const float *conv_w;     /* [conv_dim][d_conv]; tap k multiplies token t + k - (d_conv - 1) of the layer's order */
    const float *conv_b;     /* [conv_dim] */
    const float *dt_bias;    /* [nheads] */
    const float *A, *D;      /* [nheads]; D may not be NULL */
    const float *norm_w;     /* [d_inner], 16-byte aligned */
    const void *W_out;       /* bf16 [d_model][d_inner] */
} ssd_mixer_layer;

/* Workspace for mamba2_mixer_bidir (0 if the shape is refused).  Its first
 * 256 bytes are the status word (read with ssd_workspace_status). */
size_t ssd_mixer_workspace_bytes(const ssd_mixer_shape *shape);

/* out [batch][seqlen][d_model] (bf16) = the bidirectional mixer on u (bf16, same
 * shape).  Stream-ordered, asynchronous; the workspace status word must be
 * zero on entry (as for bidir_ssd).  SSD_ERR_UNSUPPORTED for other shapes. */
ssd_status mamba2_mixer_bidir(const ssd_mixer_shape *shape, const void *u, const ssd_mixer_layer *fwd,
                              const ssd_mixer_layer *rev, void *out, void *workspace, size_t workspace_bytes,
                              void *stream);

/* D [M][N] = A [M][K] W [N][K]^T on the tensor core: bf16 in and out, float32
 * accumulation; M a multiple of 128, K of 64, N of 8.  The workspace is the
 * 256-byte status area (zero on entry). */
ssd_status ssd_gemm_bf16(int M, int N, int K, const void *A, const void *W, void *D, void *workspace,
                         size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * The attention mixer of DiffuMamba-H.
 *
 * "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", technical
 * summary section 2: DiffuMamba-H inserts one Transformer block (an attention
 * mixer) after every five Mamba blocks.  The page does not spell the attention
 * out; it is read as the attention of a diffusion language model, where every
 * token sees the whole sequence (no mask):
 *
 *   O[b, i, h, :] = sum_j softmax_j(scale q[b, i, h, :] . k[b, j, h, :]) v[b, j, h, :]
 *
 * and the block around it as  out = attention(split(u W_qkv^T)) W_o^T  (no
 * bias, no positional encoding: the page names none).
 * ------------------------------------------------------------------------ */
typedef struct {
    int batch, seqlen;       /* any seqlen >= 0 for ssd_attention */
    int nheads, headdim;     /* headdim 64 or 128; batch and nheads up to 65535 */
} ssd_attn_shape;

/* out = attention(q, k, v) on the tensor core; bf16 in and out, float32 softmax
 * and accumulation.  Element d of head h of token t of sequence b is at
 * [(b seqlen + t) ld + h headdim + d] for each of q, k, v (ldq, ldk, ldv) and out
 * (ldo): row strides in elements, >= nheads*headdim and multiples of 8, so q, k
 * and v may be column blocks of one packed projection.  scale 0 means
 * 1/sqrt(headdim).  Device pointers, 16-byte aligned, owned by the caller; the
 * workspace is the 256-byte status area (zero on entry; read it with
 * ssd_workspace_status).  Stream-ordered, asynchronous.  SSD_ERR_UNSUPPORTED
 * for another headdim, SSD_ERR_INVALID_ARG for bad pointers or strides. */
ssd_status ssd_attention(const ssd_attn_shape *shape, const void *q, long long ldq, const void *k, long long ldk,
                         const void *v, long long ldv, void *out, long long ldo, float scale, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Workspace for attention_block (0 if the shape is refused): the status area,
 * the packed q/k/v projection and the attention output. */
size_t ssd_attention_block_workspace_bytes(const ssd_attn_shape *shape);

/* The attention block: qkv = u W_qkv^T (u bf16 [batch][seqlen][d_model], W_qkv
 * bf16 [3 nheads headdim][d_model], q, k, v its three column blocks in that
 * order), o = attention(q, k, v) with scale 1/sqrt(headdim), out = o W_o^T
 * (W_o bf16 [d_model][nheads headdim], out bf16 [batch][seqlen][d_model]).
 * batch*seqlen a multiple of 128, d_model of 64.  Workspace 256-byte aligned,
 * of ssd_attention_block_workspace_bytes, status word zero on entry. */
ssd_status attention_block(const ssd_attn_shape *shape, int d_model, const void *u, const void *W_qkv,
                           const void *W_o, void *out, void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BIDIR_SSD_H */
