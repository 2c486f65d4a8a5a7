/*
 * dsc.h -- C ABI of libdsc.so: the causal dynamic short convolution on NVIDIA B200
 * (sm_100a).
 *
 * The operation ("Convolucoes Curtas Dinamicas Melhoram Transformers",
 * gist.science/pt/paper/2606.03825, section "Metodologia > Convolucoes Curtas
 * Dinamicas"):
 *
 *   Mecanismo:       y_t = sum_{k=0}^{W-1} w(t)_k (.) x_{t-k}     (elementwise per channel)
 *   Posicionamento:  applied with a residual, X = X + dynamicShortConv(X)
 *   Parametrizacao:  w(t) is produced by a learned linear map of the hidden state;
 *                    (1) low-rank factorisation of rank R: w(t) = z_t U, whose second
 *                        factor the fused kernel applies on chip ("Implementacao de
 *                        Treinamento Eficiente", fused low-rank kernel), and
 *                    (2) head-wise tying: one filter is shared by G consecutive channels.
 *
 * Every entry point computes, for each sequence b, token t and channel c,
 *
 *   y[b,t,c] = x[b,t,c] + sum_{k=0}^{W-1} f(b,t,c,k) * x[b,t-k,c],   x[b,t',c] = 0 for t' < 0,
 *
 * where the tap k = 0 multiplies the current token, g(c) = floor(c / G) is the
 * filter group of channel c, and f is
 *   dsc_fwd:          w[b,t,g(c),k]                        (explicit dynamic filters)
 *   dsc_fwd_lowrank:  sum_r z[b,t,r] U[r, g(c)*W + k]      (filters formed on chip)
 *   dsc_static_fwd:   w[c,k]                               (static depthwise filters)
 * Sequences are independent: nothing crosses from one b to another.
 *
 * Conventions shared by all entry points
 *   - Layouts are dense and row-major, last index fastest:
 *       x, y, dy, dx [B,T,D];  w, dw [B,T,D/G,W];  z, dz [B,T,R];
 *       U, dU [R,(D/G)*W] with column j = g*W + k;  static w, dw [D,W].
 *   - Pointers are device memory owned by the caller; the library allocates
 *     nothing and keeps no pointer after the call returns.  Inputs are read-only.
 *     Outputs must not overlap inputs.
 *   - x, w, z, U, y, dy and dx share the element type `dt`; dz, dU and the weight
 *     gradients dw are always fp32.  Arithmetic is fp32 (fp32 accumulation); bf16
 *     outputs are rounded once, to nearest even.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 *     enqueue work on the current CUDA device.
 *   - Requirements: B, T, D, G, W >= 1, D % G == 0, 1 <= W <= 8, 1 <= R <= 256;
 *     D a multiple of 8 (bf16) or 4 (fp32); every pointer 16-byte aligned;
 *     B*T < 2^31.
 *   - Errors are reported by the return value; no exception crosses the ABI and
 *     nothing is launched when validation fails:
 *       DSC_ERR_INVALID_ARG  null pointer, non-positive size, D % G != 0;
 *       DSC_ERR_UNSUPPORTED  W or R out of range, D not a multiple of the vector
 *                            width, misaligned pointer, workspace too small;
 *       DSC_ERR_CUDA         a CUDA launch error (read from cudaGetLastError).
 *     dsc_last_error() returns a human-readable detail for the calling thread.
 *   - Results are deterministic: repeated calls on the same inputs produce
 *     bitwise-identical outputs (reductions run in a fixed order, no float atomics).
 */
#ifndef DSC_H
#define DSC_H

#include <stddef.h>

#if defined(__GNUC__)
#define DSC_API __attribute__((visibility("default")))
#else
#define DSC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSC_OK = 0,
    DSC_ERR_INVALID_ARG = 1,
    DSC_ERR_UNSUPPORTED = 2,
    DSC_ERR_CUDA = 3
} dsc_status_t;

typedef enum { DSC_F32 = 0, DSC_BF16 = 1 } dsc_dtype_t;

/* Same type as cudaStream_t. */
typedef struct CUstream_st *dsc_stream_t;

/* Forward with explicit dynamic filters (Mecanismo + Posicionamento, head-wise
 * tying by G).  x, y [B,T,D]; w [B,T,D/G,W], element (b,t,g,k) multiplies
 * x[b,t-k,c] for every channel c of group g. */
DSC_API dsc_status_t dsc_fwd(const void *x, const void *w, void *y,
                     int B, int T, int D, int G, int W,
                     dsc_dtype_t dt, dsc_stream_t stream);

/* Fused low-rank forward ("Implementacao de Treinamento Eficiente", fused low-rank
 * kernel): the filters w(t) = z_t U are formed on chip, tile by tile, and never
 * written to memory.  x, y [B,T,D]; z [B,T,R]; U [R,(D/G)*W]. */
DSC_API dsc_status_t dsc_fwd_lowrank(const void *x, const void *z, const void *U, void *y,
                             int B, int T, int D, int G, int W, int R,
                             dsc_dtype_t dt, dsc_stream_t stream);

/* Bytes of device workspace dsc_bwd_lowrank needs for these sizes (0 if none). */
DSC_API size_t dsc_bwd_lowrank_workspace_bytes(int B, int T, int D, int G, int W, int R,
                                       dsc_dtype_t dt);

/* Backward of dsc_fwd_lowrank (chain rule through Mecanismo and Parametrizacao 1):
 *   dx[b,s,c] = dy[b,s,c] + sum_{k, s+k<T} w[b,s+k,g(c),k] dy[b,s+k,c]
 *   dw[b,t,g,k] = sum_{c in g, t-k>=0} dy[b,t,c] x[b,t-k,c]      (on chip only)
 *   dz[b,t,r] = sum_j dw[b,t,j] U[r,j]
 *   dU[r,j]   = sum_{b,t} z[b,t,r] dw[b,t,j]                    (over all B*T tokens)
 * dx [B,T,D] has type dt; dz [B,T,R] and dU [R,(D/G)*W] are fp32 and are
 * overwritten, not accumulated.  `workspace` is caller-owned device scratch of at
 * least dsc_bwd_lowrank_workspace_bytes() bytes (may be NULL when that is 0); its
 * contents on entry do not matter. */
DSC_API dsc_status_t dsc_bwd_lowrank(const void *x, const void *z, const void *U, const void *dy,
                             void *dx, float *dz, float *dU,
                             void *workspace, size_t workspace_bytes,
                             int B, int T, int D, int G, int W, int R,
                             dsc_dtype_t dt, dsc_stream_t stream);

/* Backward of dsc_fwd (explicit filters): dx [B,T,D] of type dt and the per-token
 * filter gradient dw [B,T,D/G,W] in fp32 (overwritten). */
DSC_API dsc_status_t dsc_bwd(const void *x, const void *w, const void *dy,
                     void *dx, float *dw,
                     int B, int T, int D, int G, int W,
                     dsc_dtype_t dt, dsc_stream_t stream);

/* Static depthwise causal convolution, the primitive the method generalises
 * ("Declaracao do Problema"): y = x + conv(x; w), w [D,W] fixed over t. */
DSC_API dsc_status_t dsc_static_fwd(const void *x, const void *w, void *y,
                            int B, int T, int D, int W,
                            dsc_dtype_t dt, dsc_stream_t stream);

/* Bytes of device workspace dsc_static_bwd needs for these sizes. */
DSC_API size_t dsc_static_bwd_workspace_bytes(int B, int T, int D, int W, dsc_dtype_t dt);

/* Backward of dsc_static_fwd: dx [B,T,D] of type dt, and dw [D,W] fp32 summed over
 * all B*T tokens in a fixed order (overwritten). */
DSC_API dsc_status_t dsc_static_bwd(const void *x, const void *w, const void *dy,
                            void *dx, float *dw,
                            void *workspace, size_t workspace_bytes,
                            int B, int T, int D, int W,
                            dsc_dtype_t dt, dsc_stream_t stream);

/* dsc_static_bwd without a caller-provided workspace.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory, such as a
 * plug-in that a host framework hands only its input and output buffers, or a
 * latency-critical loop that must not call cudaMalloc (which can synchronise the
 * device).  It computes exactly what dsc_static_bwd computes, with the same arguments
 * minus the workspace, and allocates nothing.
 *   - Scratch comes from one fixed array of dsc_static_bwd_noalloc_max_scratch_bytes()
 *     (16 MiB) compiled into the library; every GPU that loads the library holds it
 *     until the process exits.  Sizes whose dsc_static_bwd_workspace_bytes() exceed it
 *     are rejected with DSC_ERR_UNSUPPORTED and a message naming both sizes.
 *   - Each call looks up the array's device address (cudaGetSymbolAddress) with the
 *     calling device current, so the address stays right if the device's context is
 *     reset.  The first call on a device may load the library's module onto it; make
 *     that first call before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's contents.
 *     Calls that can overlap on the GPU (other streams, other host threads) race on
 *     it; the caller must order them.  No part of it needs to start at zero. */
DSC_API dsc_status_t dsc_static_bwd_noalloc(const void *x, const void *w, const void *dy,
                                            void *dx, float *dw,
                                            int B, int T, int D, int W,
                                            dsc_dtype_t dt, dsc_stream_t stream);

/* Size in bytes of the fixed scratch array dsc_static_bwd_noalloc uses. */
DSC_API size_t dsc_static_bwd_noalloc_max_scratch_bytes(void);

/* One decode step for B sequences: the single new token x_t of each sequence, with its
 * W-1 previous inputs held in a caller-owned rolling window (inference, which the page
 * leaves to further engineering: "Significancia e Alegacoes").  For each b and c,
 *   y_t[b,c] = x_t[b,c] + sum_{k=0}^{W-1} f(b,c,k) * x_{t-k}[b,c],
 * where x_{t-k} for k >= 1 is row W-1-k of state[b] and f is
 *   dsc_decode_step:          w_t[b, g(c), k]                    (explicit filters)
 *   dsc_decode_step_lowrank:  sum_r z_t[b,r] U[r, g(c)*W + k]    (w_t = z_t U)
 * Afterwards state[b] holds the window of the next step: its rows moved up by one and
 * x_t in the last row (updated in place).
 *   x_t, y_t [B,D];  w_t [B,D/G,W];  z_t [B,R];  U [R,(D/G)*W];
 *   state [B,W-1,D], row 0 the oldest input; a sequence starts from a zeroed window
 *   (inputs before its start count as zero, as in the forward).  state may be NULL
 *   when W = 1.  Stepping a sequence from a zero window reproduces the forward's
 *   outputs token by token.
 * Same element type, alignment and error rules as the other entry points; no two of
 * y_t, x_t and state may overlap.  dsc_decode_step_lowrank forms w_t on the tensor cores
 * (the fused forward's kernel, one row per sequence) for bf16 shapes that kernel takes,
 * else on CUDA cores; it returns DSC_ERR_UNSUPPORTED when R and W are too large for the
 * CUDA-core shared-memory tile (R = 256 with W = 8). */
DSC_API dsc_status_t dsc_decode_step(const void *x_t, const void *w_t, void *state, void *y_t,
                                     int B, int D, int G, int W,
                                     dsc_dtype_t dt, dsc_stream_t stream);
DSC_API dsc_status_t dsc_decode_step_lowrank(const void *x_t, const void *z_t, const void *U,
                                             void *state, void *y_t,
                                             int B, int D, int G, int W, int R,
                                             dsc_dtype_t dt, dsc_stream_t stream);

/* The low-rank op followed by rotary position embedding (RoPE) of its output, fused:
 * the convolution sits on the Q, K and V projections before RoPE ("Metodologia >
 * Convolucoes Curtas Dinamicas > Posicionamento"), so with the projections stacked as
 * [Q | K | V] along D the first n_rot channels (Q and K) of y = x + conv(x) are rotated
 * before y is stored, and the backward takes the gradient of the rotated output.
 * RoPE in its original form: within each head of dh channels, channel pair (2i, 2i+1)
 * of token t (its position in the sequence) is rotated by the angle of pair i,
 *   y'[2i] = y[2i] cos - y[2i+1] sin,   y'[2i+1] = y[2i] sin + y[2i+1] cos,
 * with (cos, sin) read from the caller's table cs.
 *   cs     fp32 [dh/2, T, 2], 16-byte aligned: (cos, sin) of pair i at position t is
 *          cs[(i*T + t)*2 + 0..1] (pair-major, so that a warp's consecutive tokens read
 *          contiguous bytes)
 *   dh     head size, a multiple of 16;  n_rot a multiple of dh, 0 <= n_rot <= D
 *   dsc_fwd_lowrank_rope: as dsc_fwd_lowrank, y rotated on its first n_rot channels;
 *   dsc_bwd_lowrank_rope: as dsc_bwd_lowrank with dy_rot the gradient of the rotated
 *     output: dy = RoPE^T(dy_rot) is formed in shared memory (rounded to the element
 *     type once) and never written to HBM; same workspace as dsc_bwd_lowrank.
 * Only sizes on the tensor-core path (dsc_lowrank_path() == 3) are taken; others get
 * DSC_ERR_UNSUPPORTED.  n_rot = 0 is the plain op. */
DSC_API dsc_status_t dsc_fwd_lowrank_rope(const void *x, const void *z, const void *U, const float *cs,
                                          void *y, int B, int T, int D, int G, int W, int R,
                                          int dh, int n_rot, dsc_dtype_t dt, dsc_stream_t stream);
DSC_API dsc_status_t dsc_bwd_lowrank_rope(const void *x, const void *z, const void *U, const float *cs,
                                          const void *dy_rot, void *dx, float *dz, float *dU,
                                          void *workspace, size_t workspace_bytes,
                                          int B, int T, int D, int G, int W, int R,
                                          int dh, int n_rot, dsc_dtype_t dt, dsc_stream_t stream);

/* Sequence sharding (a sequence of length P*T split into P consecutive shards of T
 * tokens, one per rank).  Each rank calls dsc_fwd_lowrank / dsc_bwd_lowrank on its own
 * shard, which treats the shard as a whole sequence, and then the matching halo call
 * below on the same stream.  The causal window reaches W-1 tokens back ("Metodologia:
 * Mecanismo"), so only W-1 rows per sequence differ from the unsharded result:
 *   dsc_fwd_lowrank_halo: recomputes y rows t < min(W-1, T) with x[t-k], t-k < 0, read
 *     from x_prev (overwrites those rows of y);
 *   dsc_bwd_lowrank_halo: recomputes dx rows t >= T-(W-1) with dy[t+k] and
 *     w[t+k] = z[t+k] U, t+k >= T, read from dy_next / z_next (overwrites those rows of
 *     dx), and adds to dz rows t < W-1 and to dU the filter-gradient terms
 *     dw[t,g,k] = sum_{c in g} dy[t,c] x_prev[W-1+t-k, c] for k > t that the shard's call
 *     could not see (dz and dU are accumulated in fp32, not overwritten).
 *   x_prev  [B, W-1, D]: the W-1 tokens just before the shard (row 0 the oldest), or
 *           NULL for the first shard (nothing to do: the zero padding is right);
 *   dy_next [B, W-1, D], z_next [B, W-1, R]: the W-1 tokens just after the shard, or
 *           both NULL for the last shard;
 *   the other arguments, shapes and types are those of the shard's own call (T is the
 *   shard length, any T >= 1; when T < W-1 the halos span several shards and the caller
 *   assembles them).  dU is this rank's: summing it over the ranks (and over data-
 *   parallel replicas) is the caller's collective.  Deterministic: fixed summation
 *   orders, no atomics.  DSC_ERR_INVALID_ARG if exactly one of dy_next / z_next is NULL. */
DSC_API dsc_status_t dsc_fwd_lowrank_halo(const void *x, const void *z, const void *U,
                                          const void *x_prev, void *y,
                                          int B, int T, int D, int G, int W, int R,
                                          dsc_dtype_t dt, dsc_stream_t stream);
DSC_API dsc_status_t dsc_bwd_lowrank_halo(const void *x_prev, const void *z, const void *U,
                                          const void *dy, const void *dy_next, const void *z_next,
                                          void *dx, float *dz, float *dU,
                                          int B, int T, int D, int G, int W, int R,
                                          dsc_dtype_t dt, dsc_stream_t stream);

/* Which implementations the low-rank entry points use for these sizes: bit 0 set when
 * dsc_fwd_lowrank runs on the tensor-core (tcgen05) kernel, bit 1 when
 * dsc_bwd_lowrank does; 0 = both on CUDA cores; -1 = invalid sizes.  The tensor-core
 * kernels take bf16 with R in {16, 32, 64}, D a multiple of 64, G a power of two
 * <= 64 and (64/G)*W a multiple of 8; other valid sizes run on CUDA cores. */
DSC_API int dsc_lowrank_path(int B, int T, int D, int G, int W, int R, dsc_dtype_t dt);

/* Diagnostic: the current device's fault word.  A tensor-core kernel that waited past
 * its time limit (one second per wait) records a nonzero code here and returns early,
 * leaving its outputs undefined.  Synchronous (copies from the device); reset != 0
 * clears the word afterwards. */
DSC_API unsigned dsc_device_fault(int reset);

/* Test hook for the tensor-core kernels' bounded waits; not for production use.  Arms
 * the next dsc_fwd_lowrank or dsc_bwd_lowrank call on this host thread that runs on the
 * tensor-core kernels: in that launch every wait gives up after wait_limit_us
 * microseconds, and one CTA withholds the loads of its first tile, so that a wait does
 * run out.  The call returns DSC_OK, its outputs are undefined, and dsc_device_fault()
 * then reports a nonzero code; nothing faults or hangs, and later calls run normally.
 * The hook exists so that the give-up-and-clean-up path can be tested. */
DSC_API void dsc_test_arm_wait_timeout(unsigned wait_limit_us);

/* Static description of a status code. */
DSC_API const char *dsc_status_string(dsc_status_t status);

/* Detail of the last failed call on this host thread ("" if none). */
DSC_API const char *dsc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DSC_H */
