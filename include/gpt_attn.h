/*
 * gpt_attn -- causal multi-head scaled-dot-product attention for NVIDIA B200
 * (sm_100a), forward and backward, behind a plain C ABI.
 *
 * The operation ("NanoGPT Speedrun baseline", section "El Mecanismo de
 * Atencion"): for every batch b and head h (heads are an extra batch
 * dimension, as in the GPT-2 lecture's attention module),
 *
 *     O = softmax(scale * Q K^T) V,   with key j blocked for query i when j > i
 *
 * (the boolean triu(diagonal=1) mask of "Un GPT desde cero + nanoGPT",
 * Laboratorio L2.1, True = blocked; blocked scores are -inf before the
 * softmax, so each row renormalises over its visible keys).  With a window
 * W >= 1, key j is visible to query i iff i - W < j <= i (the long/short
 * sliding-window attention of the modded-nanogpt README's technique list).
 * The backward pass is the exact gradient of sum(O * dO).
 *
 * Conventions shared by every entry point:
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are bf16, contiguous [B, H, T, D]
 *     (row-major, D fastest), in device memory owned by the caller.
 *   - lse is fp32 [B, H, T]: lse[i] = ln sum_{visible j} exp(scale * q_i . k_j),
 *     the natural-log row log-sum-exp.  Written by the forward pass, read by
 *     the backward pass.
 *   - D must be 64 or 128.  T >= 1, B >= 1, H >= 1; B*H*T*D must fit in int64.
 *   - Every device pointer must be 16-byte aligned (the TMA rule).
 *   - window <= 0 means plain causal; window >= T is the same as causal.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     only enqueue work: there is no host synchronisation and no allocation.
 *   - Errors are returned as gpt_attn_status codes; no exceptions, no abort.
 *     After an error the outputs are unspecified.  Kernels never hang: every
 *     wait inside them is bounded, and a wait that runs out records
 *     GPT_ATTN_ERR_TIMEOUT in a per-device status word read by gpt_attn_check.
 */
#ifndef GPT_ATTN_H
#define GPT_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPT_ATTN_OK = 0,
    GPT_ATTN_ERR_NULL = 1,            /* a required pointer is NULL */
    GPT_ATTN_ERR_SHAPE = 2,           /* B, H or T < 1, or B*H*T*D overflows */
    GPT_ATTN_ERR_UNSUPPORTED_D = 3,   /* D is not 64 or 128 */
    GPT_ATTN_ERR_ALIGN = 4,           /* a pointer is not 16-byte aligned */
    GPT_ATTN_ERR_CUDA = 5,            /* a CUDA call or kernel launch failed */
    GPT_ATTN_ERR_TIMEOUT = 6,         /* a device-side bounded wait ran out */
    GPT_ATTN_ERR_WORKSPACE = 7,       /* backward workspace missing or too small */
    GPT_ATTN_ERR_UNAVAILABLE = 8,     /* not available in this build (debug-only entry points) */
    GPT_ATTN_ERR_BOUNDS = 9           /* debug build: a kernel's bounds check failed (access skipped) */
} gpt_attn_status;

/*
 * Forward pass.  Computes O and lse as defined above.
 *   q, k, v : const bf16 [B, H, T, D], device.
 *   o       : bf16 [B, H, T, D], device, written.
 *   lse     : fp32 [B, H, T], device, written.
 *   scale   : multiplier of the scores; 1/sqrt(D) gives the softmax(QK^T/sqrt(d_k))
 *             of the definition (d_k read as the head dimension).
 *   window  : <= 0 causal; >= 1 sliding window of that many keys (diagonal included).
 * Returns GPT_ATTN_OK or an error code.  Asynchronous on `stream`.
 */
int gpt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int T, int D, float scale, int window, void* stream);

/*
 * Which keys each query sees, for the *_ex entry points: the long/short
 * sliding-window pattern and the document-aligned training batches of the
 * modded-nanogpt README's technique list, in this library's reading.  Key j
 * is visible to query i of head (b, h) iff
 *     j <= i,  and  i - j < W_h when W_h >= 1,  and  j >= doc_start[b][i],
 * where W_h = head_windows[h] if head_windows is given, else `window`
 * (<= 0 for either means no window), and doc_start[b][i] is the first
 * position of the document holding token i (0 everywhere when doc_start is
 * NULL: the row is one document).
 *   window       : window of every head when head_windows is NULL.
 *   head_windows : HOST memory, H ints, read during the call (a per-layer
 *                  pattern is one call per layer with its own window; a
 *                  window warm-up is a different window per step).  At most
 *                  64 heads, else GPT_ATTN_ERR_SHAPE.
 *   doc_start    : DEVICE memory, int32 [B, T], 4-byte aligned, owned by the
 *                  caller and read by the kernels.  Valid contents: for every
 *                  row, doc_start[i] <= i, non-decreasing in i, and either
 *                  doc_start[i] = i (a document starts) or doc_start[i] =
 *                  doc_start[i-1].  Values are clamped to [0, i], so other
 *                  contents cannot make a kernel read out of bounds, but give
 *                  unspecified results.
 */
typedef struct {
    int window;
    const int* head_windows;
    const int* doc_start;
} gpt_attn_mask;

/*
 * Element strides of one bf16 tensor indexed [b, h, t, d] with d contiguous
 * (stride 1): the address of element (b, h, t, d) is base + b*batch + h*head
 * + t*token + d.  Contiguous [B, H, T, D] is {H*T*D, T*D, D}; the q, k and v
 * of a fused projection output [B, T, 3, H, D] are {3*T*H*D, D, 3*H*D} from
 * base + {0, 1, 2}*H*D ("heads as a batch dimension" without a transpose, as
 * the GPT-2 lecture's attention module lays them out).  Every stride must be
 * a multiple of 8 elements (16 bytes, the TMA rule), else GPT_ATTN_ERR_ALIGN;
 * negative strides give GPT_ATTN_ERR_SHAPE.  Tensors written by a call must
 * not overlap.
 */
typedef struct {
    long long batch, head, token;
} gpt_attn_strides;

/* The layouts of every tensor of a forward or backward call. */
typedef struct {
    gpt_attn_strides q, k, v, o;       /* forward and backward */
    gpt_attn_strides dO, dq, dk, dv;   /* backward only (ignored by the forward) */
} gpt_attn_layout;

/*
 * gpt_attn_fwd with the visibility of `mask` (NULL: plain causal) and the
 * tensor layouts of `layout` (NULL: every tensor contiguous [B, H, T, D]).
 * Same arguments, ownership and errors as gpt_attn_fwd, plus
 * GPT_ATTN_ERR_SHAPE for per-head windows with H > 64 and GPT_ATTN_ERR_ALIGN
 * for a doc_start not 4-byte aligned or a stride not a multiple of 8.  lse
 * stays contiguous [B, H, T].  gpt_attn_fwd(..., window, ...) is this call
 * with {window, NULL, NULL} and NULL.
 */
int gpt_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int T, int D, float scale, const gpt_attn_mask* mask,
                    const gpt_attn_layout* layout, void* stream);

/*
 * Bytes of device workspace gpt_attn_bwd needs for this shape: an fp32 dQ
 * accumulator [B, H, T, D], three 32-bit row vectors per head padded to a
 * multiple of 128 rows (the log2-scaled lse, Delta_i = dO_i . O_i, and the
 * rows' lower key bounds under a document mask), one int per (head, 128-key
 * tile), and 16 bytes for the work-unit counter of the backward kernel:
 * 4 * (B*H*T*D + 3*B*H*T_pad + B*H*T_pad/128) + 16 with
 * T_pad = ceil(T / 128) * 128.  Returns 0 for shapes gpt_attn_bwd would reject.
 */
size_t gpt_attn_bwd_workspace_bytes(int B, int H, int T, int D);

/*
 * Backward pass of L = sum(O * dO).
 *   q, k, v, o, dO : const bf16 [B, H, T, D], device (o and lse from gpt_attn_fwd
 *                    with the same q, k, v, scale and window).
 *   lse            : const fp32 [B, H, T], device.
 *   dq, dk, dv     : bf16 [B, H, T, D], device, written.
 *   workspace      : device buffer of at least gpt_attn_bwd_workspace_bytes(B,H,T,D)
 *                    bytes, 16-byte aligned, owned by the caller; its contents on
 *                    entry are ignored and on return are unspecified.
 * The dQ contributions of the key tiles are added into the fp32 accumulator by
 * bulk reductions whose order varies between runs, so dQ may differ in the last
 * bits; dK, dV and the forward pass are deterministic.  The workspace also holds
 * the backward kernel's work-unit counter: backward calls whose work may overlap
 * on the GPU need distinct workspaces.
 * Returns GPT_ATTN_OK or an error code.  Asynchronous on `stream`.
 */
int gpt_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dO, void* dq, void* dk, void* dv,
                 int B, int H, int T, int D, float scale, int window,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * gpt_attn_bwd with the visibility of `mask` (NULL: plain causal) and the
 * layouts of `layout` (NULL: contiguous); o and lse must come from
 * gpt_attn_fwd_ex with the same mask.  Same arguments and errors as
 * gpt_attn_bwd and gpt_attn_fwd_ex.  Runs the three stages below in order
 * (the separate stage entry points take contiguous tensors and a window).
 */
int gpt_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                    const float* lse, const void* dO, void* dq, void* dk, void* dv,
                    int B, int H, int T, int D, float scale, const gpt_attn_mask* mask,
                    const gpt_attn_layout* layout, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * The three stages gpt_attn_bwd runs, in this order, exposed so callers can
 * schedule or time them separately.  Same arguments, layouts, ownership and
 * error codes as gpt_attn_bwd; the workspace must be the same buffer for all
 * three calls of one backward pass.
 *
 * gpt_attn_bwd_delta: Delta_i = dO_i . O_i and the log2-scaled lse into the
 *   workspace rows, and zeroes the workspace's fp32 dQ accumulator.
 *   Memory-bound.
 * gpt_attn_bwd_grads: the tensor-core pass over (batch*head, 128-key tile):
 *   writes dK and dV, and adds every dQ contribution into the fp32
 *   accumulator.
 * gpt_attn_bwd_dq_convert: dQ = bf16(scale * accumulator) (the accumulator
 *   holds dS K; `scale` must be the one passed to gpt_attn_bwd_grads).
 */
int gpt_attn_bwd_delta(const void* o, const float* lse, const void* dO, int B, int H, int T, int D,
                       void* workspace, size_t workspace_bytes, void* stream);
int gpt_attn_bwd_grads(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                       int B, int H, int T, int D, float scale, int window,
                       void* workspace, size_t workspace_bytes, void* stream);
int gpt_attn_bwd_dq_convert(void* dq, int B, int H, int T, int D, float scale,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * gpt_attn_bwd without a caller-supplied workspace, for callers that cannot
 * allocate device memory at the point where they run the backward pass: for
 * example code running inside an engine's enqueue step or a host callback,
 * where cudaMalloc is not allowed, or a process whose device memory is owned
 * entirely by a pooling allocator that must not be bypassed.  (The pages
 * describe no such entry point; this is a library convenience.)
 *
 * The workspace is a fixed array inside the library, 32 MiB (33554432 bytes)
 * per GPU, created when the library is loaded on that GPU and kept until the
 * process exits.  Shapes whose gpt_attn_bwd_workspace_bytes(B,H,T,D) exceeds
 * 32 MiB are rejected with GPT_ATTN_ERR_WORKSPACE (for example B=8, H=12,
 * T=1024, D=64 fits; B=64, H=12, T=1024, D=64 does not).  Nothing is
 * allocated or freed: no cudaMalloc, no cudaFree.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on a device share the one array, so
 * calls whose work overlaps on the GPU (different streams, or several host
 * threads) race with each other: serialise them, e.g. on one stream.
 * Arguments, layouts, results and the other error codes are those of
 * gpt_attn_bwd.  Asynchronous on `stream`.
 */
int gpt_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv,
                         int B, int H, int T, int D, float scale, int window, void* stream);

/*
 * Decode attention: one new query per (batch, head) against its cached keys
 * and values, the inner step of the generation loop of "Un GPT desde cero +
 * nanoGPT" (Laboratorio L2.1, generate): the model is rerun on the growing
 * sequence and only the last position is kept, so the result equals the last
 * row of the causal forward over the sequence so far.  Sequence b holds L_b =
 * seq_lens[b] tokens (clamped to [0, T_max]) and its query is the last one; it
 * sees keys j < L_b, and with window >= 1 only j >= L_b - window.
 *   q            : const bf16 [B, H, D], device (the new token's query).
 *   k_cache,
 *   v_cache      : const bf16 [B, H, T_max, D], device; rows >= L_b are not read.
 *   seq_lens     : const int32 [B], DEVICE memory (so the call can be captured
 *                  once and replayed as sequences grow), 4-byte aligned.
 *   o            : bf16 [B, H, D], device, written; lse: fp32 [B, H] (natural
 *                  log), device, 4-byte aligned.  A sequence with L_b = 0 gets
 *                  o = 0 and lse = -inf.
 *   workspace    : device, >= gpt_attn_decode_workspace_bytes(B, H, T_max, D,
 *                  window) bytes, 16-byte aligned (fp32 partial results of the
 *                  key splits); contents ignored on entry.
 * Memory-bound: the caches are read once.  Errors as for gpt_attn_fwd, plus
 * GPT_ATTN_ERR_WORKSPACE.  Asynchronous on `stream`.
 */
size_t gpt_attn_decode_workspace_bytes(int B, int H, int T_max, int D, int window);
int gpt_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* seq_lens,
                    void* o, float* lse, int B, int H, int T_max, int D, float scale, int window,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * QK-Norm + rotary prologue of q and k (the step before attention in the
 * modded-nanogpt README's "modernised architecture" item: rotary embeddings
 * and QK-Norm; no formulas are given there, this is the reading taken).  For
 * each row x (D values) of head (b, h) at token t:
 *     n = x / max(|x|, 1e-12)                    if qk_norm, else n = x
 *     y[i]       = n[i] cos a_i - n[i + D/2] sin a_i      (i < D/2)
 *     y[i + D/2] = n[i] sin a_i + n[i + D/2] cos a_i,     a_i = t * rope_base^(-2i/D)
 * (rope_base <= 1: no rotation).  q_raw, k_raw: const bf16; q_out, k_out:
 * bf16, written; all [B, H, T, D]-indexed with the strides strides[0..3]
 * (q_raw, k_raw, q_out, k_out; NULL: all contiguous), e.g. q_raw and k_raw as
 * the columns of a fused [B, T, 3, H, D] projection and q_out, k_out
 * contiguous inputs of gpt_attn_fwd.  Memory-bound; fp32 arithmetic.
 * Errors as for gpt_attn_fwd_ex.  Asynchronous on `stream`.
 */
int gpt_attn_qk_prologue_fwd(const void* q_raw, const void* k_raw, void* q_out, void* k_out,
                             int B, int H, int T, int D, int qk_norm, float rope_base,
                             const gpt_attn_strides* strides, void* stream);

/*
 * Gradient of gpt_attn_qk_prologue_fwd: from dq_out, dk_out (the gradients
 * of q_out, k_out, e.g. from gpt_attn_bwd) and the raw rows, writes
 * dq_raw, dk_raw: dn = R^T dy (rotated back), then dx = (dn - n (n . dn)) / |x|
 * under qk_norm.  strides[0..5]: q_raw, k_raw, dq_out, dk_out, dq_raw,
 * dk_raw (NULL: all contiguous).
 */
int gpt_attn_qk_prologue_bwd(const void* q_raw, const void* k_raw, const void* dq_out,
                             const void* dk_out, void* dq_raw, void* dk_raw, int B, int H, int T,
                             int D, int qk_norm, float rope_base, const gpt_attn_strides* strides,
                             void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word: GPT_ATTN_OK, or GPT_ATTN_ERR_TIMEOUT if a kernel's bounded wait ran
 * out since the last check, or GPT_ATTN_ERR_CUDA if a CUDA error is pending.
 * Blocking: keep it out of timed regions.
 */
int gpt_attn_check(void* stream);

/* A static, human-readable name for a status code (never NULL). */
const char* gpt_attn_status_string(int status);

/*
 * Counters of the host-side tensor-map cache.  Every call encodes the TMA
 * descriptors of its tensors from (base address, element type, B*H, T, D);
 * an encoded descriptor depends on nothing else, so the library keeps the
 * last 64 in host memory and repeated calls on the same buffers skip the
 * encoding.  Reports the lookups served from the cache, the encodings done,
 * and the entries held (any pointer may be NULL).  Host only, thread-safe.
 */
void gpt_attn_tmap_cache_stats(long long* hits, long long* misses, int* entries);

/*
 * Debug builds only (libgpt_attn_debug.so, compiled with -DGPT_ATTN_DEBUG):
 * makes the next kernels' producers skip one load, so that the attention
 * kernels' own bounded waits run out and their abort path is exercised:
 *   which = 1 : the forward producer of CTA 0 skips its first K/V tile;
 *   which = 2 : the backward producer of CTA 0 skips its first Q/dO tile;
 *   which = 0 : no skip (normal operation).
 * A skipped load is neither issued nor announced to its barrier, so nothing
 * is left in flight: the consumer's wait runs out after the wait limit
 * (GPT_ATTN_WAIT_TIMEOUT_MS), every role of the CTA leaves its loop, the
 * producer waits (bounded) for the loads it did issue, TMEM is released, and
 * gpt_attn_check reports GPT_ATTN_ERR_TIMEOUT; the context stays usable.
 * Debug builds also check TMA coordinates and TMEM column ranges before each
 * access and record GPT_ATTN_ERR_BOUNDS (skipping the access) instead of
 * issuing a bad one.  Release builds return GPT_ATTN_ERR_UNAVAILABLE.
 */
int gpt_attn_debug_skip_load(int which);

/*
 * Diagnostic: launches one small kernel that waits on a shared-memory
 * barrier nothing ever arrives at, with a bound of `timeout_us` microseconds.
 * The wait runs out, the kernel records GPT_ATTN_ERR_TIMEOUT in the status
 * word and returns normally, leaving the context usable.  It exists so tests
 * can show that the bounded waits end instead of hanging; no attention
 * kernel is involved.  Asynchronous on `stream`.
 */
int gpt_attn_debug_wait_timeout(int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT_ATTN_H */
