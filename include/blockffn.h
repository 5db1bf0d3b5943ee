/*
 * blockffn.h — C ABI of the B200 (sm_100a) BlockFFN chunk-layer forward.
 *
 * The operation (BlockFFN, as described by the lsdiaocha.cn BlockFFN article, sections 2 and 4, and the
 * BlockFFN abstract on arxivdaily 2507.08771): for a chunk of L consecutive tokens x_t (the chunk a
 * speculative-decoding verification step feeds in),
 *   s_{t,i} = x_t . Wr[:,i] + b_i                        router projection (b = 0 unless given)
 *   r_{t,i} = g_i relu(s_{t,i}) / sqrt(mean_i relu(s_{t,i})^2)    ReLU + RMSNorm router (section 2);
 *                                                        r_t = 0 when no s_{t,i} is positive
 *   U       = { i : s_{t,i} > 0 for some t }            the chunk's union of active experts (section 4)
 *   y_t     = sum_{i in U} r_{t,i} W2_i Swish(W1_i x_t)   non-gated Swish MLP experts (section 2);
 *                                                        Swish(u) = u / (1 + e^-u)
 * Only the experts in U are read from memory and evaluated.
 *
 * Layouts (row-major, no padding):
 *   x   bf16 [L, d]           Wr fp32 [d, E]      g fp32 [E]       br fp32 [E]
 *   W1  bf16 [E, de, d]       W2 bf16 [E, d, de]
 *   y   fp32 [L, d]           active_idx int32 [E]   n_active int32 [1]
 *   tok_mask uint32 [L, ceil(E/32)]  (bit i%32 of word i/32 of row t = 1 iff s_{t,i} > 0)
 *   counts int32 [2]  = { number of (t,i) with s_{t,i} <= 0,  number of experts outside U }
 *   r_out fp32 [L, E]
 *
 * Ownership and execution: every pointer argument is a DEVICE pointer owned by the caller; the
 * library keeps none of them after the call returns. Work is enqueued on `stream` (a cudaStream_t,
 * NULL = the legacy default stream) and the call returns without synchronising; outputs are valid
 * once the stream has reached the enqueued work. y is fully overwritten (rows of tokens with no
 * active expert are exactly 0). active_idx[0 .. n_active) lists U in ascending order; entries past
 * n_active are unspecified. n_active stays on the device.
 *
 * Requirements, checked before anything is enqueued (BFFN_EINVAL otherwise):
 *   1 <= L, 1 <= E <= 1024, d >= 8 and d % 8 == 0, de >= 8 and de % 8 == 0 (a row of x, W1 or W2
 *   is then a whole number of 16-byte pieces, as the bulk copies need);
 *   x, Wr, W1, W2 16-byte aligned (they are read with bulk copies), a workspace 256-byte aligned,
 *   every other pointer 4-byte aligned; required pointers non-NULL.
 * Paths: L <= 32 runs the decode path (the union's weights streamed from HBM once for the whole chunk,
 * memory-bound, deterministic: y is bit-identical run to run); chunks of up to 8 tokens use warp MMAs,
 * chunks of 9 to 32 tokens the tcgen05 tensor cores. Larger L runs the prefill path (tokens
 * grouped per active expert, grouped GEMMs on the tcgen05 tensor cores); it additionally needs d and de
 * multiples of 64, de <= 256 and y 16-byte aligned, and it adds each (token, expert) row into y with
 * hardware reductions, so y may differ in the last bits between runs (masks, union, counts and r do
 * not). A shape a path cannot take returns BFFN_EUNSUPPORTED (nothing is enqueued).
 *
 * Errors: BFFN_ECUDA when a CUDA call fails (the CUDA error is cleared); BFFN_ENOMEM when the
 * internal workspace cannot be allocated. Device-side waits are bounded (about 2 s); a wait that
 * runs out records an error in the workspace instead of hanging, which blockffn_device_status
 * reports as BFFN_ETIMEOUT.
 */
#ifndef BLOCKFFN_H
#define BLOCKFFN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BFFN_API __attribute__((visibility("default")))
#else
#define BFFN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  BFFN_OK = 0,
  BFFN_EINVAL = 1,       /* bad argument: nothing was enqueued */
  BFFN_ECUDA = 2,        /* a CUDA runtime call failed */
  BFFN_ENOMEM = 3,       /* workspace allocation failed or the given workspace is too small */
  BFFN_ETIMEOUT = 4,     /* a bounded device-side wait ran out (reported by blockffn_device_status) */
  BFFN_EUNSUPPORTED = 5  /* valid arguments, but no path of this build takes the shape */
};

/* Path selection for blockffn_chunk_forward_ex's `flags` (low two bits). */
enum { BFFN_PATH_AUTO = 0, BFFN_PATH_DECODE = 1, BFFN_PATH_PREFILL = 2 };

/* Concurrency hint in `flags` bits 4-7 (decode path): k in 1..15 (0 = 1).  The call's persistent expert
 * kernel then takes 1/k of the GPU's SMs, so that k calls for independent chunks, issued on k streams
 * with k different workspaces, run side by side and one chunk's fixed latencies (router, pipeline fill,
 * the up-projection's grid barrier) overlap another chunk's weight streaming.  At most k such calls may
 * be in flight at once.  The results do not depend on k. */
#define BFFN_FLAGS_SHARE(k) ((int)(k) << 4)

/* Fault injection for tests of the error path (decode path only; off unless this bit is set): the
 * call's router barrier waits for one CTA more than the launch has and gives up after 1 ms, as a wait
 * whose peer never arrives would.  Every CTA then records the timeout, skips the rest of its work and
 * exits; y, active_idx and the other outputs are left unspecified, blockffn_device_status reports
 * BFFN_ETIMEOUT, and the next call on the same workspace runs normally.  Nothing faults or hangs. */
#define BFFN_FLAG_INJECT_ROUTER_TIMEOUT 0x100

/* Router variant (every path; blockffn_chunk_forward_ex and blockffn_chunk_forward_batch): the ReMoE
 * router, with the sum of the ReLU outputs as the normaliser instead of their RMS (intelliparadigm survey,
 * section 5.1: gate G = ReLU(x W_g), output sum_i G_i Expert_i(x) / sum_i G_i; the BlockFFN article, section
 * 2, compares BlockFFN's RMSNorm router against it):
 *   r_{t,i} = g_i relu(s_{t,i}) / sum_i relu(s_{t,i})      (r_t = 0 when no s_{t,i} is positive)
 * The active sets, union and counts are those of the RMSNorm router; only r, and so y, change. */
#define BFFN_FLAG_ROUTER_SUM_NORM 0x200

/* Cache policy for cross-chunk expert reuse (per-chunk decode path, blockffn_chunk_forward_ex): the
 * active experts' weights are read with the L2 evict-last policy instead of evict-first, so that a next
 * call that activates the same experts (the next chunk of the same sequence at the same layer; the
 * BlockFFN article, section 5, finds most experts shared by consecutive tokens) can find them in L2.  It
 * pays only when that next call comes before other traffic has pushed them out (an L2 of 126 MB; one
 * layer's union of 20-40 experts of 2-4 MiB fits).  Results do not depend on it. */
#define BFFN_FLAG_KEEP_EXPERTS_IN_L2 0x400

/*
 * The layer forward over one chunk, with no router bias.  Uses a per-device workspace that the
 * library allocates on the first call (and grows when a later call needs more); make that first
 * call before capturing the stream into a CUDA graph.  Calls that share the internal workspace must
 * be ordered (one stream, or synchronised streams).
 */
BFFN_API int blockffn_chunk_forward(const void* x, int L, int d, const float* Wr, const float* g,
                           const void* W1, const void* W2, int E, int de, float* y,
                           int32_t* active_idx, int32_t* n_active, void* stream);

/*
 * The same with optional inputs and outputs:
 *   br        router bias fp32 [E], or NULL for none
 *   tok_mask  per-token active-expert bit mask out, or NULL
 *   counts    int32[2] out (zero router entries, experts outside the union), or NULL
 *   r_out     router output r fp32 [L, E] out, or NULL
 *   flags     BFFN_PATH_* (0 = choose by L)
 *   workspace caller-owned device scratch of at least blockffn_workspace_size(L, d, E, de) bytes,
 *             zero-filled before its first use (blockffn_workspace_init), or NULL to use the
 *             library's per-device workspace.  Two calls may run concurrently only with
 *             different workspaces.
 */
BFFN_API int blockffn_chunk_forward_ex(const void* x, int L, int d, const float* Wr, const float* g,
                              const void* W1, const void* W2, int E, int de, float* y,
                              int32_t* active_idx, int32_t* n_active, const float* br,
                              uint32_t* tok_mask, int32_t* counts, float* r_out, int flags,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace a call with these sizes needs (0 for invalid sizes). */
BFFN_API size_t blockffn_workspace_size(int L, int d, int E, int de);

/* Zero-fill a caller-owned workspace on `stream` (required once before its first use). */
BFFN_API int blockffn_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the device error word of `workspace` (NULL = the
 * library's workspace of the current device).  Returns BFFN_OK, BFFN_ETIMEOUT when a bounded
 * device wait ran out since the last check, BFFN_EINVAL when a batched call met a layer index outside
 * [0, n_layers), or BFFN_ECUDA.
 */
BFFN_API int blockffn_device_status(void* workspace, void* stream);

/*
 * Many independent chunks in one call: the batched decode path (lsdiaocha.cn BlockFFN article,
 * sections 2, 4 and 7: per chunk the same router, union and sparse experts as blockffn_chunk_forward;
 * the chunks may belong to different sequences of one serving step, or to different layers of a
 * stacked model whose weights are stored one layer after another).
 *   x           bf16 [C, L, d]            C chunks of L tokens (1 <= L <= 8)
 *   layer       int32 [C] on the device: the weight set of each chunk, or NULL for chunk c -> c % n_layers.
 *               An index outside [0, n_layers) leaves that chunk empty (n_active 0, y 0) and makes
 *               blockffn_device_status report BFFN_EINVAL.
 *   Wr          fp32 [n_layers, d, E]     g fp32 [n_layers, E]     br fp32 [n_layers, E] or NULL
 *   W1          bf16 [n_layers, E, de, d] W2 bf16 [n_layers, E, d, de]
 *   y           fp32 [C, L, d]            active_idx int32 [C, E]   n_active int32 [C]
 *   counts      int32 [C, 2] or NULL      tok_mask uint32 [C, L, ceil(E/32)] or NULL
 *   flags       BFFN_FLAGS_SHARE(k): the GPU's SMs form k teams (default min(8, C)); team i takes chunks
 *               i, i + k, i + 2k, ... in order, and the next chunk's weights stream while the current
 *               chunk finishes, so no SM idles between chunks.
 *   workspace   at least blockffn_batch_workspace_size(C, L, d, E, de, flags) bytes, or NULL for the
 *               library's per-device workspace (the same rules as blockffn_chunk_forward_ex).
 * Two launches are enqueued: a router kernel (one CTA per chunk) and a persistent expert kernel.  The
 * expert kernel needs the GPU's SMs to itself while it runs (its teams wait on one another with bounded
 * waits).  Results equal blockffn_chunk_forward's within the layer's tolerance (the sums run in another
 * order); the union, masks and counts are identical; y is bit-identical run to run.  L > 8, or shapes
 * whose per-CTA tiles do not fit, return BFFN_EUNSUPPORTED before anything is enqueued.
 */
BFFN_API int blockffn_chunk_forward_batch(const void* x, int C, int L, int d, const int32_t* layer,
                                          int n_layers, const float* Wr, const float* g, const float* br,
                                          const void* W1, const void* W2, int E, int de, float* y,
                                          int32_t* active_idx, int32_t* n_active, int32_t* counts,
                                          uint32_t* tok_mask, int flags, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* Bytes of workspace a blockffn_chunk_forward_batch call with these sizes and flags needs (0 if invalid). */
BFFN_API size_t blockffn_batch_workspace_size(int C, int L, int d, int E, int de, int flags);

/*
 * Cross-chunk expert reuse (the BlockFFN article, section 5: most experts a token activates are active for
 * the next one as well).  For c < C: overlap[c] = |U_a(c) ∩ U_b(c)|, the experts in both chunk c's union
 * of call a and chunk c's union of call b, given as the active lists and counts those calls wrote
 * (active_idx [C, E] with the first n_active[c] entries of row c ascending, n_active [C]; all device
 * memory).  The reuse rate of chunk c is overlap[c] / n_active_b[c].  One small kernel on `stream`;
 * BFFN_EINVAL for bad sizes or pointers (4-byte alignment, non-NULL), BFFN_ECUDA for a launch failure.
 * Entries outside [0, E) are ignored.
 */
BFFN_API int blockffn_union_overlap(const int32_t* active_idx_a, const int32_t* n_active_a,
                                    const int32_t* active_idx_b, const int32_t* n_active_b, int C, int E,
                                    int32_t* overlap, void* stream);

/*
 * The layer's backward (the training side of the layer computed by blockffn_chunk_forward, RMSNorm router;
 * lsdiaocha.cn BlockFFN article, section 2 gives the forward; the backward is its chain rule).  For T tokens
 * x (bf16 [T, d]) and upstream gradient dy (fp32 [T, d], 16-byte aligned) of y:
 *   dx fp32 [T, d], dWr fp32 [d, E], db fp32 [E], dg fp32 [E], dW1 fp32 [E, de, d], dW2 fp32 [E, d, de]
 * are written (overwritten), with Wr fp32 [d, E], br fp32 [E] or NULL, g fp32 [E], W1 bf16 [E, de, d],
 * W2 bf16 [E, d, de] as in the forward.  A token whose router outputs are all zero has r = 0 and passes no
 * gradient to the router.  Only the (token, expert) pairs whose router pre-activation is positive are
 * evaluated (every other pair's terms are exact zeros through a = 0 and r = 0): they are grouped by expert
 * on the device and every expert contraction runs over its own pairs; every contraction runs on the warp
 * tensor cores, fp32 operands carried as bf16 hi + lo pairs, with fp32 accumulation in a fixed order
 * (bit-identical reruns).
 * workspace: device memory of at least blockffn_layer_backward_workspace_size(T, d, E, de) bytes, 256-byte
 * aligned (about 12 T E de + 4 T E d bytes, sized for every pair active; its contents need not be
 * initialised).
 * Requirements (BFFN_EINVAL otherwise): T >= 1, T <= 8 388 480, d and de multiples of 8, 1 <= E <= 1024,
 * T E de < 2^31, T d < 2^31;
 * x, W1, W2, dy 16-byte aligned, the rest 4-byte aligned, non-NULL except br.  A smaller workspace returns
 * BFFN_ENOMEM, a failed launch BFFN_ECUDA.
 */
BFFN_API int blockffn_layer_backward(const void* x, int T, int d, const float* Wr, const float* br, const float* g,
                                     const void* W1, const void* W2, int E, int de, const float* dy, float* dx,
                                     float* dWr, float* db, float* dg, float* dW1, float* dW2, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Bytes of workspace blockffn_layer_backward needs (0 if the sizes are invalid). */
BFFN_API size_t blockffn_layer_backward_workspace_size(int T, int d, int E, int de);

/*
 * Low-bit expert weights (not a BlockFFN claim: the intelliparadigm survey, section 4.1, lists low-bit
 * quantisation of MoE expert weights; the layer computed is unchanged, lsdiaocha.cn BlockFFN article,
 * sections 2 and 4).  Format, for NE = n_layers * E experts (layer l owns experts l E .. l E + E - 1):
 *   W1[e][j][k] = s1[e][j] * e4m3(q1[e][j][k])            one power-of-two scale per row of W1
 *   W2[e][k][j] = t2[l] * s2[e][j] * e4m3(q2[e][k][j])    one per column of W2, as the layer's largest
 *                                                         power of two t2[l] times a ratio s2 <= 1
 * e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, largest finite value 448.  A row's (column's)
 * scale is the smallest 2^m with 448 * 2^m >= its largest |w|; a code is w / 2^m rounded to the nearest
 * e4m3 value, ties to even.  Every dequantised weight is exactly a bf16 value.
 *
 * blockffn_quantize_fp8: W1 bf16 [NE, de, d], W2 bf16 [NE, d, de] -> W1q uint8 [NE, de, d], W2q uint8
 * [NE, d, de], s1 fp32 [NE, de], s2 fp32 [NE, de], t2 fp32 [n_layers].  Device pointers; W1, W2, W1q, W2q
 * 16-byte aligned, the rest 4-byte aligned; d, de multiples of 16.  Six kernels on `stream`.
 */
BFFN_API int blockffn_quantize_fp8(const void* W1, const void* W2, int n_layers, int E, int d, int de,
                                   uint8_t* W1q, uint8_t* W2q, float* s1, float* s2, float* t2, void* stream);

/*
 * The batched decode forward (as blockffn_chunk_forward_batch: C chunks of up to 8 tokens, the same router,
 * union, r, y, masks and counts) on fp8 expert weights in the format above.  The expert weights stream at
 * one byte each: an up-projection kernel per 64 rows of an active expert's W1 and an output-stationary
 * down-projection kernel per 64 rows of y, both converting the codes to f16 for the warp tensor cores
 * (x is converted to f16 too: |x| must stay below 65504).  y is bit-reproducible.
 *   flags: BFFN_FLAG_ROUTER_SUM_NORM or 0.
 *   workspace: at least blockffn_batch_fp8_workspace_size(C, L, d, E, de) bytes (256-byte aligned), or
 *   NULL for the library's per-device workspace.
 * Requirements as blockffn_chunk_forward_batch, plus d and de multiples of 16 (BFFN_EINVAL otherwise).
 */
BFFN_API int blockffn_chunk_forward_batch_fp8(const void* x, int C, int L, int d, const int32_t* layer,
                                              int n_layers, const float* Wr, const float* g, const float* br,
                                              const uint8_t* W1q, const float* s1, const uint8_t* W2q,
                                              const float* s2, const float* t2, int E, int de, float* y,
                                              int32_t* active_idx, int32_t* n_active, int32_t* counts,
                                              uint32_t* tok_mask, int flags, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* Bytes of workspace blockffn_chunk_forward_batch_fp8 needs (0 if the sizes are invalid). */
BFFN_API size_t blockffn_batch_fp8_workspace_size(int C, int L, int d, int E, int de);

/*
 * The CLS-aware training objectives and their backward through the router (lsdiaocha.cn BlockFFN article,
 * section 3: an activation-locality loss, a binary cross-entropy between adjacent tokens' activation
 * patterns compared through LeftShift, the patterns approximated by a sharp sigmoid; and a
 * chunk-sparsification loss, the probability that an expert is activated by at least one token of a
 * chunk of L consecutive tokens, minimised).  With s = x Wr + br and p = sigmoid(alpha s):
 *   L_AL = mean over chunks c, adjacent pairs (t, t+1) of the chunk and experts i of
 *          BCE(p_{c,t,i}; q = p_{c,t+1,i}) = -(q log p + (1 - q) log(1 - p))   (0 when L = 1)
 *   L_CS = mean over chunks c and experts i of 1 - prod_t (1 - p_{c,t,i})
 *   J    = w_al L_AL + w_cs L_CS;  the gradient flows through both sides of each pair.
 *   x     bf16 [C * L, d], the chunks one after another       Wr fp32 [d, E]    br fp32 [E] or NULL
 *   loss  fp32 [2] out: { L_AL, L_CS } (unweighted)
 *   dS    fp32 [C * L, E] out: dJ/ds (also the call's scratch for s)
 *   dWr   fp32 [d, E] out: x^T dS, or NULL     db fp32 [E] out: sum_t dS, or NULL
 *   dx    fp32 [C * L, d] out: dS Wr^T (this term of the input gradient, overwritten), or NULL
 *   workspace  device memory of at least blockffn_cls_losses_workspace_size(C, L, d, E) bytes, 256-byte
 *              aligned, owned by the caller; its contents need not be initialised.
 * All pointers are DEVICE pointers; work is enqueued on `stream` (six kernel launches, fewer without
 * dx or dWr) and the call returns without synchronising.  Results are bit-identical run to run (every
 * sum runs in a fixed order).  The products run on the bf16 tensor cores with fp32 operands carried as
 * hi + lo bf16 pairs (about 2^-17 relative), accumulated in fp32.
 * Requirements (BFFN_EINVAL otherwise, nothing enqueued): C, L >= 1, C * L <= 2^30, d >= 8, d % 8 == 0,
 * 1 <= E <= 1024, alpha > 0 and finite, w_al and w_cs finite; x and dx 16-byte aligned, every other
 * array 4-byte aligned; x, Wr, loss, dS and workspace non-NULL.  L > 128 returns BFFN_EUNSUPPORTED;
 * a workspace smaller than needed BFFN_ENOMEM; a failed launch BFFN_ECUDA.
 */
BFFN_API int blockffn_cls_losses(const void* x, int C, int L, int d, const float* Wr, const float* br, int E,
                                 float alpha, float w_al, float w_cs, float* loss, float* dS, float* dWr,
                                 float* db, float* dx, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace blockffn_cls_losses needs for these sizes (0 if the sizes are invalid). */
BFFN_API size_t blockffn_cls_losses_workspace_size(int C, int L, int d, int E);

/*
 * blockffn_chunk_forward_noalloc — no counterpart on the BlockFFN pages; this is a deployment aid.
 *
 * The same forward as blockffn_chunk_forward (plus the optional router bias `br`, may be NULL) for
 * callers that cannot call cudaMalloc: for example a serving engine that has already reserved all
 * of device memory for weights and KV cache and hands out no scratch, or code that must not
 * synchronise the device (cudaMalloc and cudaFree may wait for outstanding GPU work).  It allocates
 * nothing: its scratch is a fixed array of BFFN_NOALLOC_SCRATCH_BYTES compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *   - Sizes whose workspace (blockffn_workspace_size) exceeds BFFN_NOALLOC_SCRATCH_BYTES return
 *     BFFN_ENOMEM before anything is enqueued.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current); make that first call before capturing the stream into a CUDA graph.
 *   - Every call on a device shares the one array and leaves its contents behind: calls whose GPU
 *     work overlaps (different streams, or several host threads) race on it and must be ordered
 *     by the caller.
 *   - It runs the decode path only: L > 32 returns BFFN_EUNSUPPORTED before anything is enqueued.
 *   - Device-side timeouts of this entry point are recorded in its own array, not in the
 *     workspace blockffn_device_status(NULL, ...) reads: blockffn_noalloc_device_status reports them.
 *   - The array's address is looked up once per device for the life of the process; resetting the
 *     device (cudaDeviceReset) and then calling this entry point again is not supported.
 * Inputs and outputs are the caller's device buffers, as for blockffn_chunk_forward.
 */
#define BFFN_NOALLOC_SCRATCH_BYTES (8u << 20)
BFFN_API int blockffn_chunk_forward_noalloc(const void* x, int L, int d, const float* Wr,
                                            const float* g, const void* W1, const void* W2, int E,
                                            int de, float* y, int32_t* active_idx,
                                            int32_t* n_active, const float* br, void* stream);

/*
 * The error check of blockffn_chunk_forward_noalloc (no counterpart on the BlockFFN pages): synchronise
 * `stream`, then read and clear the error word of the current device's compiled-in scratch array.
 * Returns BFFN_OK, BFFN_ETIMEOUT when a bounded device wait of that entry point ran out since the last
 * check, or BFFN_ECUDA.  Allocates nothing.
 */
BFFN_API int blockffn_noalloc_device_status(void* stream);

/* Static description of a status code. */
BFFN_API const char* blockffn_status_string(int status);

/* ABI version (major * 100 + minor). */
BFFN_API int blockffn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BLOCKFFN_H */
