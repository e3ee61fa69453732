/*
 * path_attn.h — C ABI of the B200 (sm_100a) PaTH attention library
 * (libpath_attn.so).
 *
 * PaTH attention ("PaTH Attention: Position Encoding via Accumulating
 * Householder Transformations"). Per head, with 0-based positions and
 *   H_s  = I - beta_s w_s w_s^T
 *        (gist.science summary, section 2 "Kernmechanisme", transition
 *         matrix; Paper-Notes page, "关键设计"),
 * the logit of query i against key j <= i is
 *   z_ij = scale * q_i^T H_i H_{i-1} ... H_{j+1} k_j + (c_i - c_j)
 *        (gist.science section 2 logit equation; Paper-Notes "整体框架"),
 * where c_t = sum_{s<=t} log f_s is the optional PaTH-FoX forget gate
 * (Paper-Notes "PaTH-FoX 扩展" equation) and 0 without it. Keys j > i are
 * masked. out_i = sum_j softmax_j(z_ij) v_j and lse_i = log sum_j exp(z_ij).
 *
 * Conventions shared by every entry point
 * - Layout: contiguous row-major. q, k, v, w, out, dout and the gradients
 *   are [B, H, L, d]; beta, log_f, lse, dbeta, dlog_f are [B, H, L] fp32.
 *   Decode tensors q, k_new, v_new, w, out are [B, H, d]; decode beta is
 *   [B, H] fp32; the caches are [B, H, capacity, d].
 * - dtype (path_dtype below) selects the element types of the d-sized
 *   tensors. beta, log_f, lse, dbeta, dlog_f are always fp32. Arithmetic
 *   accumulates in fp32; on the bf16 paths the computed boundary-adjusted
 *   queries/keys and block products are held in fp16 for the tensor-core
 *   products, which requires their entries to stay below 65504 in
 *   magnitude (true whenever |q|, |k| do and beta * |w|^2 lies in [0, 2],
 *   since then every H has norm <= 1).
 * - Pointers are DEVICE pointers unless stated otherwise. The caller owns
 *   every buffer, including the workspace; the library allocates and frees
 *   no device memory and keeps no state between calls (apart from the
 *   host-side diagnostics at the end of this header). All work is
 *   enqueued on `stream` (0 = legacy default stream); no call synchronises
 *   the host.
 * - Outputs and gradients must not alias inputs (except the decode caches,
 *   which are updated in place by design).
 * - Errors: arguments are validated on the host before anything is
 *   launched; a failed check returns a status and launches nothing. A
 *   launch failure returns PATH_ERR_CUDA (the CUDA error is left for
 *   cudaGetLastError to report as usual). No call aborts, traps or throws.
 * - Supported sizes: fwd/bwd d in {16, 32, 64, 128}; decode d in {64, 128};
 *   B, H, L >= 1; B*H*L*d < 2^40 per tensor; B*H <= 65535 and
 *   ceil(L / 128) <= 65535 (launch grid dimensions): beyond those the calls
 *   return PATH_ERR_UNSUPPORTED and the workspace queries 0.
 */
#ifndef PATH_ATTN_H
#define PATH_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *path_stream_t; /* same type as cudaStream_t */

typedef enum {
    PATH_OK = 0,
    PATH_ERR_INVALID_ARG = 1, /* null pointer, size <= 0, mismatched options */
    PATH_ERR_UNSUPPORTED = 2, /* head dim or dtype this build does not handle */
    PATH_ERR_WORKSPACE = 3,   /* workspace null or smaller than required */
    PATH_ERR_CUDA = 4,        /* a kernel launch failed */
    PATH_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (path_attn_wait_status) */
} path_status;

/*
 * Element types of one call:
 *   PATH_F32          everything fp32.
 *   PATH_BF16         q, k, v, w, out, dout, dq, dk, dv, dw (and decode
 *                     caches) bf16.
 *   PATH_BF16_F32OUT  q, k, v, w bf16; out, dout, dq, dk, dv, dw fp32
 *                     (fwd/bwd only). Use it when gradients or outputs
 *                     exceed what bf16 can hold to the needed absolute
 *                     accuracy (bf16 keeps 8 significant bits), or for the
 *                     forget-gate gradient, which depends on dout.out.
 */
typedef enum { PATH_F32 = 0, PATH_BF16 = 1, PATH_BF16_F32OUT = 2 } path_dtype;

/* Human-readable name of a status code (static storage; never NULL). */
const char *path_status_string(path_status s);

/*
 * Workspace size in bytes that path_attn_fwd (for_bwd = 0) or path_attn_bwd
 * (for_bwd != 0) needs for these sizes; 0 if the sizes are invalid or
 * unsupported. The backward size is the larger and also serves the forward.
 * The workspace is scratch (its contents on entry are ignored), except that
 * path_attn_bwd with PATH_BWD_REUSE_FWD_WORKSPACE reads what the forward left
 * in it. Alignment: 256 bytes.
 * Size: with nh = B*H, nblk = ceil(L/128) and the transported-key count
 * npairs = nblk (nblk - 1) / 2, the leading term is the stored key tiles
 * (every key block J carried to every later query block I, fp16 at bf16 inputs,
 * fp32 at fp32 inputs): nh * npairs * 128 * d * s bytes (s = 2 or 4), about
 * nh * L^2 * d * s / 256 (51.5 GB at nh = 24, L = 65536, d = 64, bf16; one
 * B200 has 180 GB). The rest grows linearly: at bf16 inputs
 * nh * (Lp * (516 + 4 d) + L * 2 d) bytes for the forward and
 * nh * (Lp * (1044 + 12 d) + L * 4 d) for the backward (block logits and their
 * adjoints, boundary-adjusted queries / keys, per-position terms, 16-bit copies
 * of v and dout; Lp = 128 nblk), plus nh * nblk * d^2 * 2 (forward) or * 6
 * (backward) for the block products and their adjoints, each buffer rounded up
 * to 256 bytes; a bf16 backward at head dim 64 or 128 also holds per-block
 * quantities of the UT transform that a forward into the same workspace leaves
 * for the adjoint, nh * nblk * 98304 bytes at d = 64 and nh * nblk * 245760 at
 * d = 128; a backward that is neither (fp32 inputs, or bf16 at head dim 16 or
 * 32) holds the per-block scratch of its closed-form adjoint, nh * nblk * (14 * 128^2 + 3 * 128 d) * 4 bytes, and a bf16 forward at
 * head dim 16 or 32 the forward part of it, nh * nblk * (7 * 128^2 + 128 d) * 4
 * bytes. At nh = 24, L = 65536, d = 64, bf16 the forward needs 53.0 GB.
 */
size_t path_attn_workspace_bytes(int B, int H, int L, int d, path_dtype dt, int for_bwd);

/*
 * Forward pass.
 * Computes out [B,H,L,d] (dtype dt) and lse [B,H,L] (fp32, natural log)
 * from q, k, v, w [B,H,L,d] (dtype dt), beta [B,H,L] (fp32, used as given:
 * the model layer's 2*sigmoid and any clipping happen before the call) and
 * the optional log_f [B,H,L] (fp32; NULL = no forget gate).
 * scale multiplies the bilinear PaTH term only; the gate is added unscaled.
 * Blockwise algorithm: per-block UT transform T^{-1} = (I + strictLower(D W
 * W^T))^{-1} D (Paper-Notes "训练策略", UT transform), boundary-adjusted
 * queries/keys per block and block products (gist.science section 3
 * "FlashAttention-Stijl Algoritme"), the full-matrix form
 * lower(QK^T) - lower(QW^T) T^{-1} strictLower(WK^T) on each diagonal block
 * (Paper-Notes "训练策略"), then online softmax and P.V.
 */
path_status path_attn_fwd(const void *q, const void *k, const void *v, const void *w,
                          const float *beta, const float *log_f, float scale, int B, int H,
                          int L, int d, path_dtype dt, void *out, float *lse, void *workspace,
                          size_t workspace_bytes, path_stream_t stream);

/* flags of path_attn_bwd */
#define PATH_BWD_REUSE_FWD_WORKSPACE 1u

/*
 * Backward pass of path_attn_fwd for the loss sum(out * dout).
 * Inputs: the forward's inputs, its out and lse, and dout [B,H,L,d].
 * Outputs: dq, dk, dv, dw [B,H,L,d] (dtype dt), dbeta [B,H,L] (fp32, w.r.t.
 * beta as passed) and, iff log_f is non-NULL, dlog_f [B,H,L] (fp32; must be
 * NULL iff log_f is NULL). Every output element is written (no accumulation
 * into existing contents). The pages state no backward; it is the chain rule
 * through the same blockwise algorithm as the forward.
 * flags: 0, or PATH_BWD_REUSE_FWD_WORKSPACE when `workspace` is the buffer
 * the matching path_attn_fwd call used (sized with for_bwd != 0 at that
 * call, and that size or more given as its workspace_bytes), holding what that
 * call left there, with q, k, w, beta and log_f unchanged since: the backward
 * then reuses the forward's block transforms and transported keys instead of
 * recomputing them. At bf16, head dims 64 and 128, the forward leaves per-block
 * quantities of the UT transform for the backward only when its workspace_bytes
 * covers the backward size; a reusing backward after a forward that was given
 * less writes no dq, dk, dw, dbeta and path_attn_wait_status reports
 * PATH_ERR_WORKSPACE. Unknown flag bits are PATH_ERR_INVALID_ARG.
 */
path_status path_attn_bwd(const void *q, const void *k, const void *v, const void *w,
                          const float *beta, const float *log_f, float scale, int B, int H,
                          int L, int d, path_dtype dt, const void *out, const float *lse,
                          const void *dout, void *dq, void *dk, void *dv, void *dw,
                          float *dbeta, float *dlog_f, unsigned flags, void *workspace,
                          size_t workspace_bytes, path_stream_t stream);

/*
 * Device-side waits of the tensor-core kernels are bounded: if one gives up
 * (a pipeline stage never completed), the kernel records it in the first
 * bytes of the workspace, writes NaN to the rows it could not finish, frees
 * its tensor memory and returns instead of hanging. This call waits for
 * `stream`, then returns PATH_ERR_TIMEOUT if the last path_attn_fwd /
 * path_attn_bwd that used `workspace` recorded such an event, PATH_ERR_WORKSPACE
 * if a reusing backward found the forward's saved quantities missing (see
 * path_attn_bwd), else PATH_OK (PATH_ERR_CUDA if the read-back itself fails).
 * It synchronises the host.
 */
path_status path_attn_wait_status(const void *workspace, path_stream_t stream);

/*
 * Workspace size in bytes for path_decode_step; 0 if invalid/unsupported.
 */
size_t path_decode_workspace_bytes(int B, int H, int capacity, int d, path_dtype dt);

/*
 * One decode step (Paper-Notes "训练策略", inference paragraph; gist.science
 * section 3 "Inferentie"): with n = n_cached valid rows in the caches,
 *   1. every cached key j < n is updated in place, k_j <- k_j - beta w (w^T k_j)
 *      (computed in fp32, stored back in dtype dt, rounded to nearest even);
 *   2. k_new / v_new are written untransformed into row n of k_cache / v_cache;
 *   3. out = softmax_j(scale * q^T k_j) V over the n+1 rows (the updated keys
 *      as stored), written to out [B,H,d].
 * After the call the caches hold n+1 rows; the caller advances n.
 * Requires 0 <= n_cached and n_cached + 1 <= capacity (else
 * PATH_ERR_INVALID_ARG). q, k_new, v_new, w: [B,H,d]; beta: [B,H] fp32.
 */
path_status path_decode_step(const void *q, const void *k_new, const void *v_new, const void *w,
                             const float *beta, float scale, int B, int H, int d, int n_cached,
                             int capacity, path_dtype dt, void *k_cache, void *v_cache, void *out,
                             void *workspace, size_t workspace_bytes, path_stream_t stream);

/*
 * path_decode_step_noalloc: the same decode step as path_decode_step (same
 * arguments and results, minus the workspace) for callers that cannot call
 * cudaMalloc: for example a caller whose device memory is entirely owned by
 * another allocator (a framework's caching allocator or a fixed pool that
 * must stay the only owner), or one that cannot afford an allocation's
 * latency or its failure in the middle of decoding. It allocates nothing:
 * the per-chunk partial results live in a fixed 4 MiB device array inside
 * the library (1,048,576 floats); every GPU that loads the library holds its
 * own copy until the process exits. The pages have no counterpart to this
 * entry point.
 * - Limit: B*H*ceil(n_cached/16384)*(d+2) <= 1,048,576; beyond that the call
 *   returns PATH_ERR_WORKSPACE and launches nothing. Within it, the rows per
 *   chunk grow (256, 1024, 4096 or 16384) until the partials fit.
 * - The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture. The
 *   address is kept for the life of the process: after cudaDeviceReset (or
 *   anything else that tears down and re-creates the device's primary context)
 *   it no longer names the array, so do not call this entry point again in a
 *   process that has reset the device.
 * - Every call on a device shares that device's array and leaves its last
 *   contents there. Nothing in it needs clearing between calls, but calls on
 *   one device whose work overlaps on the GPU (e.g. on unordered streams)
 *   race on it: order them.
 */
path_status path_decode_step_noalloc(const void *q, const void *k_new, const void *v_new,
                                     const void *w, const float *beta, float scale, int B, int H,
                                     int d, int n_cached, int capacity, path_dtype dt,
                                     void *k_cache, void *v_cache, void *out,
                                     path_stream_t stream);

/*
 * PaTH-FoX decode step: path_decode_step with the forget gate. Each cached
 * key j carries its gate bias g_j = c_t - c_j (the "PaTH-FoX 扩展" logit term
 * of the Paper-Notes page, for the position t being decoded), updated in
 * place like the keys:
 *   1. keys as in path_decode_step, and g_j <- g_j + log_f for j < n;
 *   2. k_new / v_new into row n, and g_n = 0;
 *   3. out = softmax_j(scale * q^T k_j + g_j) V over the n+1 rows.
 * log_f: [B,H] fp32, log f_t of the position being decoded (<= 0 for a
 * forget gate, not checked). g_cache: [B,H,capacity] fp32, rows 0..n-1 as
 * the previous step or path_attn_prefill left them; after the call rows
 * 0..n. The workspace is sized by path_decode_workspace_bytes. Everything
 * else, including the errors, as path_decode_step; log_f or g_cache NULL is
 * PATH_ERR_INVALID_ARG.
 */
path_status path_decode_step_gated(const void *q, const void *k_new, const void *v_new,
                                   const void *w, const float *beta, const float *log_f,
                                   float scale, int B, int H, int d, int n_cached, int capacity,
                                   path_dtype dt, void *k_cache, void *v_cache, float *g_cache,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   path_stream_t stream);

/*
 * Prefill: path_attn_fwd over positions 0..L-1 (same arguments, results and
 * workspace, sized by path_attn_workspace_bytes with for_bwd = 0 or 1), and
 * the decode cache those positions leave, ready for path_decode_step (or
 * path_decode_step_gated with the gate) at n_cached = L:
 *   k_cache row j = H_{L-1} ... H_{j+1} k_j  (the in-place key update of the
 *                   Paper-Notes "训练策略" inference paragraph, applied for
 *                   every later position; computed blockwise from the
 *                   forward's transported keys and block products),
 *   v_cache row j = v_j,
 *   g_cache row j = c_{L-1} - c_j = sum of log_f over positions j+1..L-1.
 * k_cache, v_cache: [B,H,capacity,d] in the input element type (fp32 for
 * PATH_F32, bf16 for PATH_BF16 and PATH_BF16_F32OUT), 16-byte aligned;
 * g_cache: [B,H,capacity] fp32, NULL iff log_f is NULL. Only rows 0..L-1 are
 * written. Requires d in {64, 128} (the decode head dims; else
 * PATH_ERR_UNSUPPORTED) and L <= capacity (else PATH_ERR_INVALID_ARG). The
 * caches must not alias the inputs.
 */
path_status path_attn_prefill(const void *q, const void *k, const void *v, const void *w,
                              const float *beta, const float *log_f, float scale, int B, int H,
                              int L, int d, path_dtype dt, void *out, float *lse, void *k_cache,
                              void *v_cache, float *g_cache, int capacity, void *workspace,
                              size_t workspace_bytes, path_stream_t stream);

/*
 * The w / beta prologue: the model-layer step that makes the attention's w and
 * beta from token features x (Paper-Notes "关键设计": w_t from a low-rank linear
 * layer, a short convolution with filter size 3 and L2 normalisation;
 * beta_t = 2 sigmoid(u^T x_t + b); gist.science section 2). Per sequence, position t,
 * head h, channel c of the H d channels:
 *   wt_t = (x_t A) Bw;   z_t[c] = f[c,0] wt_t[c] + f[c,1] wt_{t-1}[c] + f[c,2] wt_{t-2}[c]
 *   (wt = 0 before the sequence start);   w_t^h = z_t^h / max(|z_t^h|, 1e-6);
 *   beta_t^h = min(2 sigmoid(x_t . U[:, h] + b[h]), beta_max)
 * Layouts (row-major, contiguous): x [B,L,D]; A [D,r]; Bw [r,H*d]; U [D,H] (in the
 * input type of dt); f [H*d,3], b [H] fp32. Outputs w [B,H,L,d] (the output type of
 * dt) and beta [B,H,L] fp32: the inputs path_attn_fwd takes. beta_max in (0, 2]
 * (2: no clip; bf16 training clips, e.g. 1.99). d in {16, 32, 64, 128}.
 * The low-rank products and their adjoints run as cuBLASLt GEMMs in fp32 (TF32
 * tensor cores for bf16 inputs, which TF32 holds exactly); its scratch is part of
 * `workspace` (path_wbeta_workspace_bytes). Errors as for path_attn_fwd.
 */
size_t path_wbeta_workspace_bytes(int B, int L, int D, int r, int H, int d, path_dtype dt,
                                  int for_bwd);
path_status path_wbeta_fwd(const void *x, const void *A, const void *Bw, const float *f,
                           const void *U, const float *b, float beta_max, int B, int L, int D,
                           int r, int H, int d, path_dtype dt, void *w, float *beta,
                           void *workspace, size_t workspace_bytes, path_stream_t stream);
/*
 * Backward of sum(w * dw) + sum(beta * dbeta): dx [B,L,D] (output type of dt) and
 * the parameter gradients dA [D,r], dBw [r,H*d], df [H*d,3], dU [D,H], db [H] (fp32,
 * overwritten, summed over all B*L positions in a fixed order). dw [B,H,L,d] in the
 * output type, dbeta [B,H,L] fp32 (e.g. path_attn_bwd's dw and dbeta). beta gets no
 * gradient where the clip holds. flags: PATH_BWD_REUSE_FWD_WORKSPACE when
 * `workspace` (sized for the backward) holds the matching path_wbeta_fwd's state.
 */
path_status path_wbeta_bwd(const void *x, const void *A, const void *Bw, const float *f,
                           const void *U, const float *b, float beta_max, int B, int L, int D,
                           int r, int H, int d, path_dtype dt, const void *dw, const float *dbeta,
                           void *dx, float *dA, float *dBw, float *df, float *dU, float *db,
                           unsigned flags, void *workspace, size_t workspace_bytes,
                           path_stream_t stream);

/*
 * Diagnostics (host-side, process-wide; not needed for normal use).
 *
 * path_kernel_launch_count: number of CUDA kernels this library has launched
 * in this process so far.
 *
 * path_profile_enable(on): while on, every internal stage of an entry point
 * (UT prep, transport chain, attention main loop, ...) is bracketed by two CUDA
 * events recorded on the call's stream. Returns the previous setting. Event
 * creation is the only resource it uses; no device memory.
 *
 * path_profile_read(out, max_entries): waits for the recorded events,
 * accumulates their elapsed times per stage name into out[0..n) and returns
 * n (<= max_entries); the recorded events are released.
 */
typedef struct {
    char name[32];
    double total_ms;
    int count;
} path_stage_time;

unsigned long long path_kernel_launch_count(void);
int path_profile_enable(int on);
int path_profile_read(path_stage_time *out, int max_entries);

/*
 * Test hook for the bounded waits (process-wide, off by default; the pages have
 * no counterpart). While on (on = 1), every tensor-core path_attn_fwd (bf16
 * inputs, d = 64 or 128) makes the load producer of its last query tile skip
 * the copy of that tile's first off-diagonal key / value block (it neither
 * issues it nor announces its bytes), and every wait of that kernel gives up
 * after 2 ms instead of 0.5 s. The tile that waits for the block then gives
 * up: its rows of out and lse are written as NaN and path_attn_wait_status
 * reports PATH_ERR_TIMEOUT; the other tiles complete normally and the CUDA
 * context stays usable. The producer still waits for every copy it did issue
 * before its block exits. Needs L > 128 (at least two query tiles). Returns
 * PATH_OK, or PATH_ERR_INVALID_ARG if `on` is not 0 or 1.
 */
path_status path_test_withhold_kv_load(int on);

#ifdef __cplusplus
}
#endif

#endif /* PATH_ATTN_H */
