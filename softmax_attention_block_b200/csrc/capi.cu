// C ABI of the PaTH attention library: argument validation, workspace
// layout, and the launch sequence of each entry point.
#include <math.h>

#include "attn.cuh"
#include "attn_tc.cuh"
#include "prep.cuh"
#include "runtime.cuh"

using namespace path;

namespace {

struct Layout {
    int nh, L, d, nblk, Lp;
    long long npairs;
    size_t tsz;
};

Layout make_layout(int B, int H, int L, int d, path_dtype dt)
{
    Layout y;
    y.nh = B * H;
    y.L = L;
    y.d = d;
    y.nblk = ceil_div(L, BT);
    y.Lp = y.nblk * BT;
    y.npairs = (long long)y.nblk * (y.nblk - 1) / 2;
    y.tsz = dtype_size(types_of(dt).mid);
    return y;
}

struct AttnWs {
    int *err;  // device error word: first bounded wait that gave up (0 = none)
    float *c;
    void *Qt, *Kt, *Pm, *Khat;
    void *Vh;  // fp16 copy of v for the tensor-core forward
    float *Sd;
    PrepScratch prep;
    UtSave save;   // head dim 128, bf16, backward-sized workspace
    // backward only
    float *delta, *dQt, *dKt, *dPm, *dSd, *rowsum, *colsum;
    float *lse_p;     // lse padded to Lp (tensor-core backward)
    void *dout16;     // bf16 copy of an fp32 dout (tensor-core backward)
};

// bf16 inputs at head dim 64 take the tcgen05 UT kernels (prep_fwd_ut.cu,
// prep_bwd_ut.cu), at head dim 128 those of prep_fwd_ut128.cu and
// prep_bwd_ut128.cu; a forward into a backward-sized workspace leaves per-block
// quantities there that their adjoint reads (UtSave). Other bf16 cases take the
// closed form by batched products on the tensor cores in TF32 (prep.cu,
// gemm_tc.cu), forward and adjoint; fp32 inputs take the fp32 recurrences
// forward and the closed-form adjoint on CUDA cores (prep_fwd_rec.cu, prep.cu,
// gemm_batched.cu), which hold fp32 accuracy.
bool ut_tc_path(const Layout &y, path_dtype dt)
{
    return y.d == 64 && types_of(dt).in == BF16 && (long long)y.nh * y.nblk * BT < (1LL << 31);
}

bool ut128_path(const Layout &y, path_dtype dt)
{
    return y.d == 128 && types_of(dt).in == BF16 && (long long)y.nh * y.nblk * 2 * 128 < (1LL << 31);
}

// The single description of the workspace: used both to size and to carve it.
size_t carve_attn(void *base, const Layout &y, path_dtype dt, bool bwd, AttnWs &w)
{
    Carver c(base);
    const size_t nh = y.nh, Lp = y.Lp, d = y.d, nb = y.nblk;
    w.err = c.take<int>(64);
    w.c = c.take<float>(nh * Lp);
    w.Qt = c.take<char>(nh * Lp * d * y.tsz);
    w.Kt = c.take<char>(nh * Lp * d * y.tsz);
    w.Pm = c.take<char>(nh * nb * d * d * y.tsz);
    w.Khat = c.take<char>(nh * (size_t)y.npairs * BT * d * y.tsz);
    w.Vh = c.take<char>(nh * (size_t)y.L * d * 2);
    w.Sd = c.take<float>(nh * nb * BT * BT);
    PrepDims D{y.nh, y.L, y.d, y.nblk, types_of(dt).in, types_of(dt).out};
    // the buffers above are the forward's, at the same offsets in a forward- and a
    // backward-sized workspace (a backward may reuse the forward's); the rest only
    // the backward path that reads it gets
    // closed-form scratch: the backward's adjoint, and the forward of bf16 inputs
    // at head dims 16 and 32 (fp32 inputs take the recurrences forward)
    if (ut_tc_path(y, dt) || ut128_path(y, dt)) {
        if (bwd) carve_ut_save(c, D, w.save);
    } else if (bwd || D.dt != F32) {
        carve_prep_scratch(c, D, bwd, w.prep);
    }
    if (bwd) {
        w.delta = c.take<float>(nh * Lp);
        w.dQt = c.take<float>(nh * Lp * d);
        w.dKt = c.take<float>(nh * Lp * d);
        w.dPm = c.take<float>(nh * nb * d * d);
        w.dSd = c.take<float>(nh * nb * BT * BT);
        w.rowsum = c.take<float>(nh * Lp);
        w.colsum = c.take<float>(nh * Lp);
        w.lse_p = c.take<float>(nh * Lp);
        w.dout16 = c.take<char>(nh * (size_t)y.L * d * 2);
    }
    return c.bytes();
}

bool fwd_dims_ok(int B, int H, int L, int d)
{
    if (B <= 0 || H <= 0 || L <= 0) return false;
    const long long elems = (long long)B * H * L * d;
    return elems > 0 && elems < (1LL << 40);
}

bool head_dim_supported(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// bf16 inputs at head dims 64 and 128 go through the tcgen05 UT kernels, which
// load q, k and w by TMA: their base addresses must be 16-byte aligned.
bool tma_inputs_ok(int d, path_dtype dt, const void *q, const void *k, const void *w)
{
    if ((d != 64 && d != 128) || types_of(dt).in != BF16) return true;
    const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                         reinterpret_cast<uintptr_t>(w);
    return (al & 15u) == 0;
}

// Heads and 128-row blocks index launch grid dimensions limited to 65535.
bool grid_ok(int B, int H, int L)
{
    return (long long)B * H <= 65535 && (L + BT - 1) / BT <= 65535;
}

bool dtype_ok(path_dtype dt)
{
    return dt == PATH_F32 || dt == PATH_BF16 || dt == PATH_BF16_F32OUT;
}

bool decode_dtype_ok(path_dtype dt) { return dt == PATH_F32 || dt == PATH_BF16; }

path_status launch_status(cudaError_t e) { return e == cudaSuccess ? PATH_OK : PATH_ERR_CUDA; }

#define TRY(x)                                          \
    do {                                                \
        cudaError_t e_ = (x);                           \
        if (e_ != cudaSuccess) return PATH_ERR_CUDA;    \
    } while (0)

// Tile row coordinates of the tensor maps (int32) stay in range.
bool tc_rows_fit(const Layout &y)
{
    return (long long)y.nh * (y.npairs + 1) * BT < (1LL << 31) &&
           (long long)y.nh * y.Lp < (1LL << 31) && (long long)y.nh * y.nblk * y.d < (1LL << 31);
}

// Tensor-core forward: bf16 inputs, d in {64, 128}, 16-byte aligned v (TMA).
bool use_tc_fwd(Types t, const Layout &y, const void *v)
{
    if (!attn_fwd_tc_supported(t, y.d)) return false;
    if (reinterpret_cast<uintptr_t>(v) & 15u) return false;
    return tc_rows_fit(y);
}

// Shared by forward and backward: gate prefix, UT prep, transport chain.
path_status run_prep_and_chain(const void *q, const void *k, const void *w, const float *beta,
                               const float *log_f, const Layout &y, path_dtype dt, AttnWs &ws,
                               cudaStream_t st)
{
    if (log_f) {
        Stage s("gate_prefix", st);
        TRY(gate_prefix(log_f, ws.c, y.L, y.Lp, y.nh, st));
    }
    const Types t = types_of(dt);
    PrepDims D{y.nh, y.L, y.d, y.nblk, t.in, t.out};
    PrepInputs in{q, k, w, beta};
    PrepOutputs out{ws.Qt, ws.Kt, ws.Pm, ws.Sd, t.mid};
    {
        Stage s("ut_prep", st);
        if (ut_tc_path(y, dt) || ut128_path(y, dt)) {
            // the save word tells a backward that reuses this workspace whether the
            // per-block quantities it reads were written by this call
            const bool save = ws.save.What != nullptr;
            TRY(cudaMemsetAsync(ws.err + UT_SAVED_WORD, save ? UT_SAVED_BYTE : 0, sizeof(int), st));
            if (y.d == 64)
                TRY(prep_forward_ut(D, in, out, save ? &ws.save : nullptr, ws.err, st));
            else
                TRY(prep_forward_ut128(D, in, out, save ? &ws.save : nullptr, ws.err, st));
        } else if (D.dt != F32) {
            ws.prep.err = ws.err;
            TRY(prep_forward_gemm(D, in, out, ws.prep, st));
        } else {
            TRY(prep_forward_rec(D, in, out, st));
        }
    }
    ChainArgs ca{ws.Kt, ws.Pm, ws.Khat, y.nblk, y.nh};
    {
        Stage s("chain", st);
        if (attn_fwd_tc_supported(t, y.d) && tc_rows_fit(y))
            TRY(chain_tc(ca, y.d, ws.err, st));
        else
            TRY(chain_simt(ca, t, y.d, st));
    }
    return PATH_OK;
}

// path_attn_fwd after argument validation: carves `workspace` into ws and
// enqueues the forward.
path_status run_forward(const void *q, const void *k, const void *v, const void *w,
                        const float *beta, const float *log_f, float scale, const Layout &y,
                        path_dtype dt, void *out, float *lse, void *workspace,
                        size_t workspace_bytes, AttnWs &ws, cudaStream_t st)
{
    const size_t need = carve_attn(nullptr, y, dt, false, ws);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    // a workspace sized for the backward also receives what a backward that
    // reuses it needs beyond the forward's own buffers
    const bool for_bwd = workspace_bytes >= carve_attn(nullptr, y, dt, true, ws);
    carve_attn(workspace, y, dt, for_bwd, ws);
    TRY(cudaMemsetAsync(ws.err, 0, sizeof(int), st));
    path_status s = run_prep_and_chain(q, k, w, beta, log_f, y, dt, ws, st);
    if (s != PATH_OK) return s;
    FwdArgs a{ws.Qt, ws.Khat, v, ws.Vh, ws.Sd, log_f ? ws.c : nullptr, scale, y.L, y.nblk, y.nh, out, lse};
    const Types t = types_of(dt);
    if (use_tc_fwd(t, y, v)) {
        {
            Stage s_cv("v_to_f16", st);
            TRY(convert_to_f16(v, ws.Vh, (long long)y.nh * y.L * y.d, st));
        }
        Stage s_attn("attn_fwd", st);
        return launch_status(attn_fwd_tc(a, t, y.d, ws.err, st));
    }
    Stage s_attn("attn_fwd", st);
    return launch_status(attn_fwd_simt(a, t, y.d, st));
}

}  // namespace

extern "C" {

const char *path_status_string(path_status s)
{
    switch (s) {
    case PATH_OK: return "ok";
    case PATH_ERR_INVALID_ARG: return "invalid argument";
    case PATH_ERR_UNSUPPORTED: return "unsupported size or dtype";
    case PATH_ERR_WORKSPACE: return "workspace missing or too small";
    case PATH_ERR_CUDA: return "CUDA launch failed";
    case PATH_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

size_t path_attn_workspace_bytes(int B, int H, int L, int d, path_dtype dt, int for_bwd)
{
    if (!fwd_dims_ok(B, H, L, d) || !head_dim_supported(d) || !dtype_ok(dt) || !grid_ok(B, H, L))
        return 0;
    AttnWs w;
    return carve_attn(nullptr, make_layout(B, H, L, d, dt), dt, for_bwd != 0, w);
}

path_status path_attn_fwd(const void *q, const void *k, const void *v, const void *w,
                          const float *beta, const float *log_f, float scale, int B, int H, int L,
                          int d, path_dtype dt, void *out, float *lse, void *workspace,
                          size_t workspace_bytes, path_stream_t stream)
{
    if (!q || !k || !v || !w || !beta || !out || !lse) return PATH_ERR_INVALID_ARG;
    if (!fwd_dims_ok(B, H, L, d) || !isfinite(scale)) return PATH_ERR_INVALID_ARG;
    if (!head_dim_supported(d) || !dtype_ok(dt) || !grid_ok(B, H, L)) return PATH_ERR_UNSUPPORTED;
    if (!tma_inputs_ok(d, dt, q, k, w)) return PATH_ERR_INVALID_ARG;
    AttnWs ws;
    return run_forward(q, k, v, w, beta, log_f, scale, make_layout(B, H, L, d, dt), dt, out, lse,
                       workspace, workspace_bytes, ws, reinterpret_cast<cudaStream_t>(stream));
}

path_status path_attn_prefill(const void *q, const void *k, const void *v, const void *w,
                              const float *beta, const float *log_f, float scale, int B, int H,
                              int L, int d, path_dtype dt, void *out, float *lse, void *k_cache,
                              void *v_cache, float *g_cache, int capacity, void *workspace,
                              size_t workspace_bytes, path_stream_t stream)
{
    if (!q || !k || !v || !w || !beta || !out || !lse || !k_cache || !v_cache)
        return PATH_ERR_INVALID_ARG;
    if ((log_f == nullptr) != (g_cache == nullptr)) return PATH_ERR_INVALID_ARG;
    if (!fwd_dims_ok(B, H, L, d) || !isfinite(scale) || capacity < L) return PATH_ERR_INVALID_ARG;
    if ((d != 64 && d != 128) || !dtype_ok(dt) || !grid_ok(B, H, L)) return PATH_ERR_UNSUPPORTED;
    // 16-byte vector access of v and the caches
    const uintptr_t al = reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(k_cache) |
                         reinterpret_cast<uintptr_t>(v_cache);
    if (al & 15u) return PATH_ERR_INVALID_ARG;
    if (!tma_inputs_ok(d, dt, q, k, w)) return PATH_ERR_INVALID_ARG;
    const Layout y = make_layout(B, H, L, d, dt);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    AttnWs ws;
    path_status s = run_forward(q, k, v, w, beta, log_f, scale, y, dt, out, lse, workspace,
                                workspace_bytes, ws, st);
    if (s != PATH_OK) return s;
    CacheArgs ca{ws.Kt, ws.Khat, ws.Pm, v, log_f ? ws.c : nullptr, y.L, y.nblk, y.nh, capacity,
                 k_cache, v_cache, g_cache};
    Stage s_c("prefill_cache", st);
    return launch_status(prefill_cache(ca, types_of(dt), d, st));
}

path_status path_attn_bwd(const void *q, const void *k, const void *v, const void *w,
                          const float *beta, const float *log_f, float scale, int B, int H, int L,
                          int d, path_dtype dt, const void *out, const float *lse, const void *dout,
                          void *dq, void *dk, void *dv, void *dw, float *dbeta, float *dlog_f,
                          unsigned flags, void *workspace, size_t workspace_bytes,
                          path_stream_t stream)
{
    if (!q || !k || !v || !w || !beta || !out || !lse || !dout || !dq || !dk || !dv || !dw ||
        !dbeta)
        return PATH_ERR_INVALID_ARG;
    if ((log_f == nullptr) != (dlog_f == nullptr)) return PATH_ERR_INVALID_ARG;
    if (!fwd_dims_ok(B, H, L, d) || !isfinite(scale)) return PATH_ERR_INVALID_ARG;
    if (!head_dim_supported(d) || !dtype_ok(dt) || !grid_ok(B, H, L)) return PATH_ERR_UNSUPPORTED;
    if (!tma_inputs_ok(d, dt, q, k, w)) return PATH_ERR_INVALID_ARG;
    const Layout y = make_layout(B, H, L, d, dt);
    AttnWs ws;
    const size_t need = carve_attn(nullptr, y, dt, true, ws);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    carve_attn(workspace, y, dt, true, ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (flags & ~PATH_BWD_REUSE_FWD_WORKSPACE) return PATH_ERR_INVALID_ARG;
    TRY(cudaMemsetAsync(ws.err, 0, sizeof(int), st));
    if (!(flags & PATH_BWD_REUSE_FWD_WORKSPACE)) {
        path_status s = run_prep_and_chain(q, k, w, beta, log_f, y, dt, ws, st);
        if (s != PATH_OK) return s;
    }
    TRY(cudaMemsetAsync(ws.dPm, 0, sizeof(float) * (size_t)y.nh * y.nblk * d * d, st));
    BwdArgs a{ws.Qt,     ws.Khat,  v,        ws.Pm,  ws.Sd,  log_f ? ws.c : nullptr,
              scale,     y.L,      y.nblk,   y.nh,   out,    dout,
              lse,       ws.delta, ws.dQt,   ws.dKt, ws.dPm, ws.dSd,
              dv,        ws.rowsum, ws.colsum};
    const Types t = types_of(dt);
    const bool tc = (attn_bwd_tc_supported(t, d) || attn_bwd128_tc_supported(t, d)) && tc_rows_fit(y) &&
                    !((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(dout)) & 15u);
    if (tc) {
        {
            Stage s_d("delta", st);
            TRY(compute_delta(a, t, d, st));
            TRY(attn_bwd_tc_prepare(a, t, d, ws.lse_p, ws.dout16, st));
        }
        TRY(cudaMemsetAsync(ws.dQt, 0, sizeof(float) * (size_t)y.nh * y.Lp * d, st));
        TRY(cudaMemsetAsync(ws.rowsum, 0, sizeof(float) * (size_t)y.nh * y.Lp, st));
        Stage s_b("attn_bwd", st);
        if (d == 128)
            TRY(attn_bwd128_tc(a, t, ws.lse_p, ws.dout16, ws.err, st));
        else
            TRY(attn_bwd_tc(a, t, ws.lse_p, ws.dout16, ws.err, st));
    } else {
        TRY(attn_bwd_simt(a, t, d, st));
    }
    PrepDims D{y.nh, y.L, y.d, y.nblk, types_of(dt).in, types_of(dt).out};
    PrepInputs in{q, k, w, beta};
    PrepGrads gr{ws.dQt, ws.dKt, ws.dPm, ws.dSd, dq, dk, dw, dbeta};
    if (ut_tc_path(y, dt)) {
        Stage s("ut_adj", st);
        TRY(prep_backward_ut(D, in, gr, ws.save, ws.err + UT_SAVED_WORD, ws.err, st));
    } else if (ut128_path(y, dt)) {
        Stage s("ut_adj", st);
        TRY(prep_backward_ut128(D, in, gr, ws.save, ws.err + UT_SAVED_WORD, ws.err, st));
    } else {
        Stage s("ut_prep_bwd", st);
        ws.prep.err = ws.err;
        TRY(prep_backward(D, in, ws.prep, gr, st));
    }
    if (log_f) {
        Stage s("gate_grad", st);
        TRY(gate_grad(ws.rowsum, ws.colsum, dlog_f, y.L, y.Lp, y.nh, st));
    }
    return PATH_OK;
}

path_status path_attn_wait_status(const void *workspace, path_stream_t stream)
{
    if (!workspace) return PATH_ERR_INVALID_ARG;
    int code = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return PATH_ERR_CUDA;
    if (code == ERR_UT_NOT_SAVED) return PATH_ERR_WORKSPACE;
    return code ? PATH_ERR_TIMEOUT : PATH_OK;
}

size_t path_decode_workspace_bytes(int B, int H, int capacity, int d, path_dtype dt)
{
    if (B <= 0 || H <= 0 || capacity <= 0 || (d != 64 && d != 128) || !decode_dtype_ok(dt) ||
        !grid_ok(B, H, 1))
        return 0;
    const size_t nchunk = (size_t)ceil_div(capacity, DECODE_CHUNK);
    return align_up((size_t)B * H * nchunk * (d + 2) * sizeof(float), 256);
}

path_status path_decode_step(const void *q, const void *k_new, const void *v_new, const void *w,
                             const float *beta, float scale, int B, int H, int d, int n_cached,
                             int capacity, path_dtype dt, void *k_cache, void *v_cache, void *out,
                             void *workspace, size_t workspace_bytes, path_stream_t stream)
{
    if (!q || !k_new || !v_new || !w || !beta || !k_cache || !v_cache || !out)
        return PATH_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || capacity <= 0 || n_cached < 0 || n_cached + 1 > capacity ||
        !isfinite(scale))
        return PATH_ERR_INVALID_ARG;
    if ((d != 64 && d != 128) || !decode_dtype_ok(dt) || !grid_ok(B, H, 1)) return PATH_ERR_UNSUPPORTED;
    // 16-byte vector access of q, w and the caches
    const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(w) |
                         reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache);
    if (al & 15u) return PATH_ERR_INVALID_ARG;
    const size_t need = path_decode_workspace_bytes(B, H, capacity, d, dt);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    DecodeArgs a{q, k_new, v_new, w, beta, scale, B * H, n_cached, capacity,
                 k_cache, v_cache, out, static_cast<float *>(workspace)};
    return launch_status(decode_step(a, (int)dt, d, reinterpret_cast<cudaStream_t>(stream)));
}

path_status path_decode_step_gated(const void *q, const void *k_new, const void *v_new,
                                   const void *w, const float *beta, const float *log_f,
                                   float scale, int B, int H, int d, int n_cached, int capacity,
                                   path_dtype dt, void *k_cache, void *v_cache, float *g_cache,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   path_stream_t stream)
{
    if (!q || !k_new || !v_new || !w || !beta || !log_f || !k_cache || !v_cache || !g_cache ||
        !out)
        return PATH_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || capacity <= 0 || n_cached < 0 || n_cached + 1 > capacity ||
        !isfinite(scale))
        return PATH_ERR_INVALID_ARG;
    if ((d != 64 && d != 128) || !decode_dtype_ok(dt) || !grid_ok(B, H, 1)) return PATH_ERR_UNSUPPORTED;
    const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(w) |
                         reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache);
    if (al & 15u) return PATH_ERR_INVALID_ARG;
    const size_t need = path_decode_workspace_bytes(B, H, capacity, d, dt);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    DecodeArgs a{q, k_new, v_new, w, beta, scale, B * H, n_cached, capacity,
                 k_cache, v_cache, out, static_cast<float *>(workspace), log_f, g_cache};
    return launch_status(decode_step(a, (int)dt, d, reinterpret_cast<cudaStream_t>(stream)));
}

path_status path_decode_step_noalloc(const void *q, const void *k_new, const void *v_new,
                                     const void *w, const float *beta, float scale, int B, int H,
                                     int d, int n_cached, int capacity, path_dtype dt,
                                     void *k_cache, void *v_cache, void *out,
                                     path_stream_t stream)
{
    if (!q || !k_new || !v_new || !w || !beta || !k_cache || !v_cache || !out)
        return PATH_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || capacity <= 0 || n_cached < 0 || n_cached + 1 > capacity ||
        !isfinite(scale))
        return PATH_ERR_INVALID_ARG;
    if ((d != 64 && d != 128) || !decode_dtype_ok(dt) || !grid_ok(B, H, 1)) return PATH_ERR_UNSUPPORTED;
    const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(w) |
                         reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache);
    if (al & 15u) return PATH_ERR_INVALID_ARG;
    const int chunk = noalloc_chunk_rows(B * H, n_cached, d);
    if (chunk == 0) return PATH_ERR_WORKSPACE;  // partials exceed the fixed scratch
    float *scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return PATH_ERR_CUDA;
    DecodeArgs a{q, k_new, v_new, w, beta, scale, B * H, n_cached, capacity,
                 k_cache, v_cache, out, scratch};
    return launch_status(decode_step_noalloc(a, (int)dt, d, chunk, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
