/*
 * bdscan.h: C ABI of the block-confined bidirectional selective scan, the
 * Mamba mixer of BDLM Mamba-H, running on NVIDIA B200 (sm_100a).
 *
 * Source of the method: "Training Hybrid Block Diffusion Language Models with
 * Partial Bidirectionality" (arXiv 2607.02805).
 *   - Abstract: the reverse Mamba scan is restricted to the active denoising
 *     block, which enables exact caching across blocks.
 *   - gist.science technical summary, "Methodik" (cache-aligned objective):
 *     Mamba layers cache only forward boundary states; the reverse scan is
 *     confined to the active block, so the prefix cache depends on the clean
 *     prefix alone.
 *   - same summary, "Wesentliche Beitraege": the objects cached by the
 *     all-block training objective equal the inference-time block caches.
 *
 * The pages never write the recurrence. This library computes the standard
 * Mamba selective scan in both directions, with shared parameters:
 *   delta_t = softplus(dt_t)  (dims.dt_softplus = 1)  or  dt_t  (= 0)
 *   a_t[n]  = exp(delta_t * A[d,n]),   b_t[n] = delta_t * x_t * B_t[n]
 *   forward   h_t = a_t * h_{t-1} + b_t            (h_{-1} = h0 or the cache)
 *             y_fwd_t = sum_n C_t[n] h_t[n] + Dskip[d] x_t
 *   reverse   g_t = a_t * g_{t+1} + b_t  inside each block [jK, (j+1)K),
 *             g = 0 after the block's last token
 *             y_rev_t = sum_n C_t[n] g_t[n] + Dskip[d] x_t
 *   output    y_t = (y_fwd_t + y_rev_t) * (z ? silu(z_t) : 1)
 * (y therefore carries Dskip * x twice.) The forward state at the end of a
 * block is the cache for the next block.
 *
 * Data layout, all row-major and contiguous, on the device:
 *   x, dt, z, y   [batch, L, D]        io dtype (fp32 or bf16)
 *   B, C          [batch, L, N]        io dtype
 *   A             [D, N]               fp32 (negative for a decaying state)
 *   Dskip         [D]                  fp32
 *   h0, h_out, h_cache  [batch, D, N]  fp32
 *   boundary      [batch, L/K, D, N]   fp32, the state after each block's
 *                                      last token (the last one equals h_out)
 *
 * Conventions shared by every entry point:
 *   - All pointers are device pointers owned by the caller; the library
 *     allocates nothing and never synchronises; scratch memory, where an
 *     entry point needs it, is passed in by the caller.
 *     Work is queued on `stream` (NULL = the legacy default stream) and the
 *     call returns without waiting for it.
 *   - Every pointer must be 16-byte aligned. D must be a multiple of 8 for
 *     bf16 and of 4 for fp32; N must be 16 or 64; L must be a multiple of K.
 *     A pointer may be NULL only when its tensor has no elements (for
 *     example x when L == 0).
 *   - Arguments are checked before anything is queued. A call that returns an
 *     error has queued nothing, except BDSCAN_ERR_CUDA, which reports a failed
 *     launch (the launch error is then also left in the CUDA runtime).
 *   - Results are deterministic: the same inputs give bit-identical outputs.
 *   - Input and output buffers must not overlap, except h_cache in
 *     bdscan_commit_block, which is read and written in place.
 */
#ifndef BDSCAN_H
#define BDSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                        /* the CUDA runtime's cudaStream_t */
typedef struct CUstream_st *bdscan_stream_t;

typedef enum {
    BDSCAN_OK = 0,
    BDSCAN_ERR_INVALID_ARG = 1,  /* NULL required pointer, negative size, L % K != 0, ... */
    BDSCAN_ERR_UNSUPPORTED = 2,  /* N not 16/64, D not a multiple of the vector width,
                                    a block too long for a pass with a reverse scan */
    BDSCAN_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    BDSCAN_ERR_WORKSPACE = 4,    /* workspace missing or smaller than the size the library asks for */
    BDSCAN_ERR_CUDA = 5          /* a kernel launch failed; see bdscan_last_cuda_error() */
} bdscan_status;

typedef enum { BDSCAN_F32 = 0, BDSCAN_BF16 = 1 } bdscan_dtype;

typedef struct {
    int64_t batch;        /* independent sequences in the call */
    int64_t seqlen;       /* L, tokens in the call (block_step / commit: L == K) */
    int64_t d_inner;      /* D, channels */
    int64_t d_state;      /* N, state size per channel: 16 or 64 */
    int64_t block;        /* K, denoising block length, K >= 1, L % K == 0 */
    int32_t io_dtype;     /* bdscan_dtype of x, dt, B, C, z and y */
    int32_t dt_softplus;  /* 1: delta = softplus(dt); 0: delta = dt */
} bdscan_dims;

typedef struct {
    const void *x;        /* [batch, L, D] */
    const void *dt;       /* [batch, L, D] raw step (softplus applied in-kernel if asked) */
    const void *B;        /* [batch, L, N] */
    const void *C;        /* [batch, L, N] */
    const void *z;        /* [batch, L, D] gate input, or NULL for no gate */
    const float *A;       /* [D, N] */
    const float *Dskip;   /* [D] */
} bdscan_inputs;

/* Full-block (all-block) training pass: every block of every sequence in one
 * launch. Forward scan over all L tokens from h0 (NULL = zero state) plus the
 * block-confined reverse scan of each block; y = (y_fwd + y_rev) * gate.
 * Optional outputs: boundary states after each block (NULL = not written) and
 * the final state h_out (NULL = not written). Blocks longer than 32 tokens
 * first sweep the reverse state alone and keep its value at every 16-token
 * span start in shared memory ((ceil(K/16) - 1) x N x 128 bytes: K up to 1408
 * at N = 16 and 320 at N = 64 with bf16 I/O, 1216 and 256 with fp32), then run
 * the fused pass span by span. Where that does not fit, a two-sweep path stages
 * the block's reverse readout in shared memory instead (K <= 768); blocks too
 * long for both return BDSCAN_ERR_UNSUPPORTED.
 * Source: full-block objective, gist.science technical summary, "Methodik";
 * cache agreement, "Wesentliche Beitraege". */
int bdscan_train_blocks(const bdscan_dims *dims, const bdscan_inputs *in,
                        const float *h0, void *y, float *boundary, float *h_out,
                        bdscan_stream_t stream);

/* Forward-only scan of a clean context (the prefix operator): h_out receives
 * the final state (required); y = y_fwd * gate if y is not NULL; boundary
 * states after every K tokens if boundary is not NULL (K only matters there).
 * Source: forward-only Mamba boundary states, gist.science technical summary,
 * "Methodik". */
int bdscan_prefill(const bdscan_dims *dims, const bdscan_inputs *in,
                   const float *h0, void *y, float *h_out, float *boundary,
                   bdscan_stream_t stream);

/* Time-chunked prefill for contexts with too few channels to fill the GPU
 * (fewer (batch, 32-channel) rows than SMs, e.g. one sequence of 65,536
 * tokens x 1536 channels). Same outputs as
 * bdscan_prefill, computed in two passes over chunks of the context: pass 1
 * scans every chunk from a zero state and records its end state and the
 * product of its decays; pass 2 rescans every chunk from the state composed
 * from the chunks before it (h_c = P_{c-1} h_{c-1} + H_{c-1}), writing y, the
 * block-boundary states and h_out. The composition reassociates the
 * recurrence, so the states agree with the sequential scan within fp32
 * rounding, not bit for bit (use bdscan_prefill where the cache must equal a
 * commit chain exactly). Two exps per (token, channel, state). When a single
 * chunk already fills the device the call runs bdscan_prefill's sequential
 * scan instead (workspace size 0). The number of chunks keeps all CTAs of a
 * pass resident at once (rows x chunks <= SMs x resident CTAs per SM).
 * ws: device scratch of bdscan_prefill_chunked_workspace(dims) bytes (the
 * size depends on the current device's SM count), 16-byte aligned, owned by
 * the caller, not preserved; BDSCAN_ERR_WORKSPACE if it is missing or too
 * small. */
size_t bdscan_prefill_chunked_workspace(const bdscan_dims *dims);
int bdscan_prefill_chunked(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                           float *h_out, float *boundary, void *ws, size_t ws_bytes, bdscan_stream_t stream);

/* bdscan_prefill_chunked without a workspace argument, for callers that cannot
 * allocate device memory: code inside a framework whose memory pool owns the
 * GPU (a raw cudaMalloc there can fail or fragment the pool), and loops that
 * must not allocate between steps (cudaMalloc and cudaFree synchronise the
 * device). The paper has no counterpart; this is a library convenience.
 * Scratch is a fixed 8 MiB array in device memory that the library holds on
 * every GPU it is loaded on until the process exits; problems whose
 * bdscan_prefill_chunked_workspace(dims) exceeds 8 MiB return
 * BDSCAN_ERR_WORKSPACE (use bdscan_prefill_chunked with your own buffer);
 * the chunk plan keeps its CTAs to one wave, so on a 148-SM B200 no size
 * needs more than about 2.5 MB.
 * The first call on a device looks up the array's device address (a CUDA
 * runtime query, done once per device); make that first call before any
 * stream capture. The address is kept for the life of the process, so the
 * entry point must not be used on a device after cudaDeviceReset, nor from a
 * context other than the device's primary context (the runtime's default):
 * the library's device memory then sits at another address. All calls share the one array and it keeps whatever the
 * last call left there; nothing in it has to start at zero, because each
 * call's first pass writes every entry its second pass reads. Calls that may
 * run at the same time on the GPU (different streams with no ordering between
 * them) race on the array and must not be issued; calls on one stream are
 * safe. Outputs and status codes are those of
 * bdscan_prefill_chunked; it allocates nothing. */
int bdscan_prefill_chunked_noalloc(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                                   float *h_out, float *boundary, bdscan_stream_t stream);

/* One denoising step of the active block (dims.seqlen == dims.block): forward
 * scan resumed from h_cache plus the in-block reverse scan from zero;
 * y = (y_fwd + y_rev) * gate. h_cache is only read.
 * Source: abstract (reverse scan restricted to the active block; exact cache
 * reuse across blocks). */
int bdscan_block_step(const bdscan_dims *dims, const bdscan_inputs *in,
                      const float *h_cache, void *y, bdscan_stream_t stream);

/* Commit a finished block (dims.seqlen == dims.block) with its clean inputs:
 * h_cache is advanced in place to the forward state after the block's last
 * token. If y is not NULL it receives what bdscan_block_step would return on
 * these inputs. Source: exact caching across blocks, abstract; cache built by
 * scanning the clean prefix, gist.science technical summary, "Methodik". */
int bdscan_commit_block(const bdscan_dims *dims, const bdscan_inputs *in,
                        float *h_cache, void *y, bdscan_stream_t stream);

/* Two-stream all-block training pass (clean prefix stream + noisy active
 * blocks). The clean stream is scanned forward only, as the cached prefix
 * operator: y_clean = y_fwd * gate (NULL = not written), boundary receives the
 * state after every clean block (required: these are the caches), h_out the
 * final state (NULL = not written). Every noisy block j then resumes the
 * forward scan from the clean cache at its start (h0 for block 0; NULL = zero)
 * and adds its block-confined reverse scan: y_noisy = (y_fwd + y_rev) * gate.
 * Both streams share dims; A and Dskip are read from each stream's inputs
 * (normally the same arrays); boundary must not alias h0. Two launches on
 * `stream`, no scratch memory. With noisy == clean this is
 * bdscan_train_blocks. Source: training protocol, gist.science technical
 * summary, "Methodik" (the prefix cache is built by scanning the clean
 * prefix; block losses are computed on top of it). */
int bdscan_train_two_stream(const bdscan_dims *dims, const bdscan_inputs *clean, const bdscan_inputs *noisy,
                            const float *h0, void *y_clean, void *y_noisy, float *boundary, float *h_out,
                            bdscan_stream_t stream);

/* Full-sequence bidirectional pass (the DiffuMamba-style mixing that the
 * block-confined design replaces): forward scan over all L tokens from h0 plus
 * a reverse scan over all L tokens from zero, y = (y_fwd + y_rev) * gate
 * (required), h_out = final forward state (NULL = not written). Equal to
 * bdscan_train_blocks with K = L, for any L. Two launches and no scratch: the
 * forward pass writes y_fwd + Dskip x into y, the reverse pass adds y_rev +
 * Dskip x and applies the gate in place (so bf16 y is rounded twice).
 * dims.block must divide L (any value; only the block-free passes run).
 * Source: the full-sequence reverse scan of earlier hybrids, abstract and
 * gist.science technical summary, "Problemstellung". */
int bdscan_full_bidirectional(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                              float *h_out, bdscan_stream_t stream);

/* Gradient outputs of bdscan_train_blocks_backward (all written, none accumulated). */
typedef struct {
    void *dx;             /* [batch, L, D] io_dtype */
    void *ddt;            /* [batch, L, D] io_dtype, gradient w.r.t. the raw dt (through softplus if used) */
    void *dz;             /* [batch, L, D] io_dtype; required when inputs have z, else ignored */
    void *dB;             /* [batch, L, N] io_dtype */
    void *dC;             /* [batch, L, N] io_dtype */
    float *dA;            /* [D, N] fp32, summed over batch and tokens */
    float *dDskip;        /* [D] fp32, summed over batch and tokens */
    float *dh0;           /* [batch, D, N] fp32 gradient w.r.t. h0, or NULL */
} bdscan_grads;

/* Workspace bytes bdscan_train_blocks_backward needs for dims (0 for an
 * unsupported d_state): per-CTA partial dB / dC rows (batch x ceil(D/32) x L
 * x 2N fp32), per-row partial dA and dDskip, and for blocks longer than 8
 * tokens the forward-state checkpoints at 8-token tile starts. */
size_t bdscan_train_blocks_backward_workspace(const bdscan_dims *dims);

/* Backward pass of bdscan_train_blocks: given dy = dLoss/dy, the gradients of
 * the loss with respect to x, dt, z, B, C, A, Dskip and h0. The pages define
 * only the forward computation (full-block objective, gist.science technical
 * summary, "Methodik"); this is its exact adjoint:
 *   ds_t = dy_t gate_t; lambda_t = ds_t C_t + a_{t+1} lambda_{t+1} over the
 *   whole sequence; mu_t = ds_t C_t + a_{t-1} mu_{t-1} inside each block;
 *   db_t = lambda_t + mu_t; da_t = lambda_t h_{t-1} + mu_t g_{t+1}.
 * boundary = the block-boundary states bdscan_train_blocks wrote for the same
 * inputs and h0 ([batch, L/K, D, N]; required when L > K): the forward state
 * is recomputed from them block by block, never stored per token. Two
 * launches on `stream` (the scan, then a fixed-order reduction of the
 * partials: results are bitwise reproducible). ws: 16-byte aligned, at least
 * bdscan_train_blocks_backward_workspace(dims) bytes, contents on entry
 * ignored; dy and the gradient arrays 16-byte aligned. Any K >= 1. */
int bdscan_train_blocks_backward(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0,
                                 const float *boundary, const void *dy, const bdscan_grads *grads, void *ws,
                                 size_t ws_bytes, bdscan_stream_t stream);

/* Context-parallel prefill, for a context split into consecutive chunks (for
 * instance one per GPU, each chunk a whole number of blocks). The forward
 * recurrence h_t = a_t h_{t-1} + b_t is affine in the state, so a chunk acts on
 * its start state as h -> P h + H: P = the product of the chunk's decays a_t,
 * H = the state the chunk reaches from zero. Composing the summaries of chunks
 * 0 .. r-1 from h0 gives chunk r's start state; chunk r then runs
 * bdscan_prefill from it. The pages describe the forward-only prefix operator
 * whose block-end states are the cache (gist.science technical summary,
 * "Methodik"); splitting its scan over chunks is this library's choice. */

/* The chunk summary of in's whole context: H = forward state after the L
 * tokens from a zero state, P = product over the L tokens of exp(delta A), both
 * [batch, D, N] fp32 (written, required unless batch * D * N == 0). dims.block
 * is not used beyond the argument checks. L == 0 gives H = 0, P = 1. One launch
 * on `stream`, no scratch. */
int bdscan_chunk_summary(const bdscan_dims *dims, const bdscan_inputs *in, float *H, float *P,
                         bdscan_stream_t stream);

/* h_in = the start state of chunk `index` of `chunks`: from h0 ([count] fp32,
 * NULL = zero state), fold h = P_q * h + H_q for q = 0 .. index-1, where H_all
 * and P_all hold the chunks' summaries one after another ([chunks][count] fp32,
 * the layout of an all-gather of the per-chunk bdscan_chunk_summary outputs;
 * may be NULL when index == 0); count = batch * D * N. h_in may not alias
 * H_all or P_all. One launch on `stream`. */
int bdscan_carry_fold(int64_t chunks, int64_t index, int64_t count, const float *h0, const float *H_all,
                      const float *P_all, float *h_in, bdscan_stream_t stream);

/* Human-readable name of a bdscan_status value (static storage). */
const char *bdscan_status_string(int status);

/* Text of the CUDA error behind the calling thread's last BDSCAN_ERR_CUDA
 * (static storage; "no error" if none). */
const char *bdscan_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int bdscan_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BDSCAN_H */
