// The w / beta prologue of PaTH attention (the model-layer step that makes the
// attention's w and beta from the token features), forward and backward.
//
// Paper-Notes "关键设计": w_t comes from a low-rank linear layer, a short
// convolution with filter size 3 and L2 normalisation; beta_t = 2 sigmoid(u^T x_t + b)
// (also gist.science section 2). Per sequence, position t and head h:
//   wt_t = (x_t A) Bw                          A [D, r], Bw [r, H d]
//   z_t[c] = sum_{k<3} f[c, k] wt_{t-k}[c]     causal, wt = 0 before the start
//   w_t^h = z_t^h / max(|z_t^h|, 1e-6)
//   beta_t^h = min(2 sigmoid(x_t . u_h + b_h), beta_max)      U = [u_1 .. u_H] [D, H]
//
// The two products of the low-rank layer and their adjoints are plain GEMMs,
// run by cuBLASLt in fp32 (TF32 tensor cores when the inputs are bf16, whose
// values TF32 holds exactly; plain fp32 for fp32 inputs). The steps in between
// are this file's kernels: the convolution, the per-head normalisation and beta
// in one pass writing w [B, H, L, d] and beta [B, H, L] for the attention, and
// their adjoints (normalisation and sigmoid, the transposed convolution, the
// filter and bias gradients as deterministic two-stage sums).
#include <cublasLt.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "runtime.cuh"

namespace path {

namespace {

constexpr float NORM_EPS = 1e-6f;
constexpr size_t LT_WS_BYTES = 32u << 20;  // cuBLASLt's scratch, carved from the caller's workspace
constexpr int RED_CHUNK = 256;             // positions per partial sum of the reductions

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// dst[i * ld + col0 + j] = src[i * cols + j] as fp32 (rows x cols)
__global__ void to_f32_kernel(const void *src, int dt, long long rows, int cols, float *dst, int ld,
                              int col0)
{
    const long long n = rows * cols;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x)
        dst[(e / cols) * ld + col0 + e % cols] = load_as_f(src, dt, e);
}

// dst[e] = src[i * ld + col0 + j] stored as dt (rows x cols)
__global__ void from_f32_kernel(const float *src, int ld, int col0, long long rows, int cols, void *dst,
                                int dt)
{
    const long long n = rows * cols;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x)
        store_from_f(dst, dt, e, src[(e / cols) * ld + col0 + e % cols]);
}

struct Dims {
    int B, L, D, r, H, d;
    __host__ __device__ long long BL() const { return (long long)B * L; }
    __host__ __device__ int Hd() const { return H * d; }
    __host__ __device__ int ldys() const { return r + H; }
};

// One warp per (position p of the B L positions, head h): z of the head's d
// channels, their norm, w, and beta.
__global__ void wbeta_fwd_kernel(Dims m, const float *wt, const float *ys, const float *f,
                                 const float *bias, float beta_max, void *w, int wdt, float *beta)
{
    const long long g = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (g >= m.BL() * m.H) return;
    const long long p = g / m.H;
    const int h = (int)(g % m.H), t = (int)(p % m.L), bi = (int)(p / m.L), Hd = m.Hd();
    float z[4];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = lane + 32 * i;
        z[i] = 0.f;
        if (e < m.d) {
            const int c = h * m.d + e;
            const float *col = wt + p * Hd + c;
            float v = f[c * 3] * col[0];
            if (t >= 1) v = fmaf(f[c * 3 + 1], col[-Hd], v);
            if (t >= 2) v = fmaf(f[c * 3 + 2], col[-2 * Hd], v);
            z[i] = v;
            ss = fmaf(v, v, ss);
        }
    }
    const float inv = 1.f / fmaxf(sqrtf(warp_sum(ss)), NORM_EPS);
    const long long row = ((long long)(bi * m.H + h) * m.L + t);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = lane + 32 * i;
        if (e < m.d) store_from_f(w, wdt, row * m.d + e, z[i] * inv);
    }
    if (lane == 0) {
        const float s = ys[p * m.ldys() + m.r + h] + bias[h];
        beta[row] = fminf(2.f / (1.f + expf(-s)), beta_max);
    }
}

// One warp per (p, h): the adjoint of the normalisation, dz = (dw - w (w . dw)) / |z|
// (dw / eps where |z| <= eps), and of beta, ds = dbeta 2 sigma (1 - sigma) where the
// clip is open, into the last H columns of dys.
__global__ void wbeta_dz_kernel(Dims m, const float *wt, const float *ys, const float *f,
                                const float *bias, float beta_max, const void *dw, int dwdt,
                                const float *dbeta, float *dz, float *dys)
{
    const long long g = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (g >= m.BL() * m.H) return;
    const long long p = g / m.H;
    const int h = (int)(g % m.H), t = (int)(p % m.L), bi = (int)(p / m.L), Hd = m.Hd();
    const long long row = ((long long)(bi * m.H + h) * m.L + t);
    float z[4], gr[4];
    float ss = 0.f, zg = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = lane + 32 * i;
        z[i] = gr[i] = 0.f;
        if (e < m.d) {
            const int c = h * m.d + e;
            const float *col = wt + p * Hd + c;
            float v = f[c * 3] * col[0];
            if (t >= 1) v = fmaf(f[c * 3 + 1], col[-Hd], v);
            if (t >= 2) v = fmaf(f[c * 3 + 2], col[-2 * Hd], v);
            z[i] = v;
            gr[i] = load_as_f(dw, dwdt, row * m.d + e);
            ss = fmaf(v, v, ss);
            zg = fmaf(v, gr[i], zg);
        }
    }
    const float n = sqrtf(warp_sum(ss));
    zg = warp_sum(zg);
    const bool big = n > NORM_EPS;
    const float inv = 1.f / fmaxf(n, NORM_EPS);
    // w . dw = (z . dw) / |z|, and w = z / |z|: dz = (dw - z (z . dw) / |z|^2) / |z|
    const float along = zg * inv * inv;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = lane + 32 * i;
        if (e < m.d) dz[p * Hd + h * m.d + e] = big ? (gr[i] - z[i] * along) * inv : gr[i] * inv;
    }
    if (lane == 0) {
        const float s = ys[p * m.ldys() + m.r + h] + bias[h];
        const float sg = 1.f / (1.f + expf(-s));
        dys[p * m.ldys() + m.r + h] = 2.f * sg < beta_max ? dbeta[row] * 2.f * sg * (1.f - sg) : 0.f;
    }
}

// The transposed convolution: dwt_t[c] = sum_k f[c, k] dz_{t+k}[c] within each sequence.
__global__ void conv_adjoint_kernel(Dims m, const float *dz, const float *f, float *dwt)
{
    const int Hd = m.Hd();
    const long long n = m.BL() * Hd;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % Hd);
        const int t = (int)((i / Hd) % m.L);
        float v = f[c * 3] * dz[i];
        if (t + 1 < m.L) v = fmaf(f[c * 3 + 1], dz[i + Hd], v);
        if (t + 2 < m.L) v = fmaf(f[c * 3 + 2], dz[i + 2 * Hd], v);
        dwt[i] = v;
    }
}

// Partial sums over chunks of RED_CHUNK positions of the filter gradient
// df[c, k] = sum_t dz_t[c] wt_{t-k}[c]: part[chunk][c][k].
__global__ void df_partial_kernel(Dims m, const float *dz, const float *wt, float *part)
{
    const int Hd = m.Hd();
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Hd) return;
    const long long p0 = (long long)blockIdx.y * RED_CHUNK;
    const long long p1 = p0 + RED_CHUNK < m.BL() ? p0 + RED_CHUNK : m.BL();
    float a0 = 0.f, a1 = 0.f, a2 = 0.f;
    for (long long p = p0; p < p1; ++p) {
        const int t = (int)(p % m.L);
        const float g = dz[p * Hd + c];
        a0 = fmaf(g, wt[p * Hd + c], a0);
        if (t >= 1) a1 = fmaf(g, wt[(p - 1) * Hd + c], a1);
        if (t >= 2) a2 = fmaf(g, wt[(p - 2) * Hd + c], a2);
    }
    float *o = part + ((long long)blockIdx.y * Hd + c) * 3;
    o[0] = a0;
    o[1] = a1;
    o[2] = a2;
}

// Partial column sums of src[rows, ld] over columns [col0, col0 + ncol), chunks of RED_CHUNK rows.
__global__ void colsum_partial_kernel(const float *src, long long rows, int ld, int col0, int ncol,
                                      float *part)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= ncol) return;
    const long long r0 = (long long)blockIdx.y * RED_CHUNK;
    const long long r1 = r0 + RED_CHUNK < rows ? r0 + RED_CHUNK : rows;
    float a = 0.f;
    for (long long i = r0; i < r1; ++i) a += src[i * ld + col0 + j];
    part[(long long)blockIdx.y * ncol + j] = a;
}

// out[j] = sum_i part[i * n + j], i < nparts (fixed order)
__global__ void sum_parts_kernel(const float *part, int nparts, int n, float *out)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n) return;
    float a = 0.f;
    for (int i = 0; i < nparts; ++i) a += part[(long long)i * n + j];
    out[j] = a;
}

// ---------------------------------------------------------------------------
// cuBLASLt GEMM in row-major terms: C[M x N] = op(A) op(B), fp32 storage.
// A is stored [M x K] (ta = false) or [K x M] (ta = true) with leading dimension
// lda; B [K x N] or [N x K] likewise; C with leading dimension ldc.
// ---------------------------------------------------------------------------
cublasLtHandle_t lt_handle()
{
    static std::mutex mu;
    static cublasLtHandle_t h = nullptr;
    std::lock_guard<std::mutex> g(mu);
    if (!h && cublasLtCreate(&h) != CUBLAS_STATUS_SUCCESS) h = nullptr;
    return h;
}

bool gemm_rm(int M, int N, int K, const float *A, int lda, bool ta, const float *B, int ldb,
             bool tb, float *C, int ldc, bool tf32, void *ws, cudaStream_t st)
{
    cublasLtHandle_t lt = lt_handle();
    if (!lt) return false;
    // column-major view: C^T [N x M] = op(B)^T [N x K] op(A)^T [K x M]
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    bool ok = cublasLtMatmulDescCreate(&op, tf32 ? CUBLAS_COMPUTE_32F_FAST_TF32 : CUBLAS_COMPUTE_32F,
                                       CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
    const cublasOperation_t opa = tb ? CUBLAS_OP_T : CUBLAS_OP_N, opb = ta ? CUBLAS_OP_T : CUBLAS_OP_N;
    ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &opa, sizeof(opa)) ==
                   CUBLAS_STATUS_SUCCESS;
    ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &opb, sizeof(opb)) ==
                   CUBLAS_STATUS_SUCCESS;
    // stored (column-major) shapes: the first operand is B's storage, the second A's
    ok = ok && cublasLtMatrixLayoutCreate(&la, CUDA_R_32F, tb ? K : N, tb ? N : K, ldb) ==
                   CUBLAS_STATUS_SUCCESS;
    ok = ok && cublasLtMatrixLayoutCreate(&lb, CUDA_R_32F, ta ? M : K, ta ? K : M, lda) ==
                   CUBLAS_STATUS_SUCCESS;
    ok = ok && cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, N, M, ldc) == CUBLAS_STATUS_SUCCESS;
    ok = ok && cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS;
    const size_t wsb = LT_WS_BYTES;
    ok = ok && cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                                    &wsb, sizeof(wsb)) == CUBLAS_STATUS_SUCCESS;
    cublasLtMatmulHeuristicResult_t heur;
    int nres = 0;
    ok = ok && cublasLtMatmulAlgoGetHeuristic(lt, op, la, lb, lc, lc, pref, 1, &heur, &nres) ==
                   CUBLAS_STATUS_SUCCESS && nres > 0;
    const float one = 1.f, zero = 0.f;
    ok = ok && cublasLtMatmul(lt, op, &one, B, la, A, lb, &zero, C, lc, C, lc, &heur.algo, ws, wsb,
                              st) == CUBLAS_STATUS_SUCCESS;
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (lc) cublasLtMatrixLayoutDestroy(lc);
    if (lb) cublasLtMatrixLayoutDestroy(lb);
    if (la) cublasLtMatrixLayoutDestroy(la);
    if (op) cublasLtMatmulDescDestroy(op);
    count_launches();
    return ok;
}

// Workspace of one call (the forward's part first, so that a backward can reuse it).
struct WbWs {
    float *x32, *wau, *bw32, *ys, *wt;
    void *lt;
    float *dz, *dwt, *dys, *dwau, *dx32, *dfpart, *dbpart;
};

int nchunks(long long rows) { return (int)((rows + RED_CHUNK - 1) / RED_CHUNK); }

size_t carve(void *base, const Dims &m, bool bwd, WbWs &w)
{
    Carver c(base);
    const size_t BL = m.BL(), D = m.D, r = m.r, H = m.H, Hd = m.Hd(), ldys = m.ldys();
    w.x32 = c.take<float>(BL * D);
    w.wau = c.take<float>(D * ldys);
    w.bw32 = c.take<float>(r * Hd);
    w.ys = c.take<float>(BL * ldys);
    w.wt = c.take<float>(BL * Hd);
    w.lt = c.take<char>(LT_WS_BYTES);
    if (bwd) {
        w.dz = c.take<float>(BL * Hd);
        w.dwt = c.take<float>(BL * Hd);
        w.dys = c.take<float>(BL * ldys);
        w.dwau = c.take<float>(D * ldys);
        w.dx32 = c.take<float>(BL * D);
        w.dfpart = c.take<float>((size_t)nchunks(BL) * Hd * 3);
        w.dbpart = c.take<float>((size_t)nchunks(BL) * H);
    }
    return c.bytes();
}

bool dims_ok(const Dims &m)
{
    if (m.B <= 0 || m.L <= 0 || m.D <= 0 || m.r <= 0 || m.H <= 0) return false;
    if (m.d != 16 && m.d != 32 && m.d != 64 && m.d != 128) return false;
    // GEMM dimensions and leading dimensions are int; rows of the reductions fit the grid
    return m.BL() * (m.D > m.Hd() ? m.D : m.Hd()) < (1LL << 31) && m.D * (long long)m.ldys() < (1LL << 31) &&
           (long long)m.r * m.Hd() < (1LL << 31) && nchunks(m.BL()) <= 65535;
}

unsigned grid_for(long long n, int per_block = 256)
{
    const long long g = (n + per_block - 1) / per_block;
    return (unsigned)(g < 148 * 64 ? (g > 0 ? g : 1) : 148 * 64);
}

// The forward's products: x32, [A | U], Bw in fp32; ys = x [A | U]; wt = ys[:, :r] Bw.
path_status forward_products(const void *x, const void *A, const void *Bw, const void *u,
                             const Dims &m, Types t, const WbWs &w, cudaStream_t st)
{
    const bool tf32 = t.in != F32;
    const int ldys = m.ldys();
    to_f32_kernel<<<grid_for(m.BL() * m.D), 256, 0, st>>>(x, t.in, m.BL(), m.D, w.x32, m.D, 0);
    to_f32_kernel<<<grid_for((long long)m.D * m.r), 256, 0, st>>>(A, t.in, m.D, m.r, w.wau, ldys, 0);
    to_f32_kernel<<<grid_for((long long)m.D * m.H), 256, 0, st>>>(u, t.in, m.D, m.H, w.wau, ldys, m.r);
    to_f32_kernel<<<grid_for((long long)m.r * m.Hd()), 256, 0, st>>>(Bw, t.in, m.r, m.Hd(), w.bw32,
                                                                     m.Hd(), 0);
    count_launches(4);
    if (cudaGetLastError() != cudaSuccess) return PATH_ERR_CUDA;
    if (!gemm_rm((int)m.BL(), ldys, m.D, w.x32, m.D, false, w.wau, ldys, false, w.ys, ldys, tf32,
                 w.lt, st))
        return PATH_ERR_CUDA;
    if (!gemm_rm((int)m.BL(), m.Hd(), m.r, w.ys, ldys, false, w.bw32, m.Hd(), false, w.wt, m.Hd(),
                 tf32, w.lt, st))
        return PATH_ERR_CUDA;
    return PATH_OK;
}

bool wbeta_dtype_ok(path_dtype dt)
{
    return dt == PATH_F32 || dt == PATH_BF16 || dt == PATH_BF16_F32OUT;
}

}  // namespace

}  // namespace path

using namespace path;

extern "C" {

size_t path_wbeta_workspace_bytes(int B, int L, int D, int r, int H, int d, path_dtype dt,
                                  int for_bwd)
{
    const Dims m{B, L, D, r, H, d};
    if (!dims_ok(m) || !wbeta_dtype_ok(dt)) return 0;
    WbWs w;
    return carve(nullptr, m, for_bwd != 0, w);
}

path_status path_wbeta_fwd(const void *x, const void *A, const void *Bw, const float *f,
                           const void *u, const float *b, float beta_max, int B, int L, int D,
                           int r, int H, int d, path_dtype dt, void *w, float *beta,
                           void *workspace, size_t workspace_bytes, path_stream_t stream)
{
    if (!x || !A || !Bw || !f || !u || !b || !w || !beta) return PATH_ERR_INVALID_ARG;
    if (!(beta_max > 0.f) || !(beta_max <= 2.f)) return PATH_ERR_INVALID_ARG;
    const Dims m{B, L, D, r, H, d};
    if (m.B <= 0 || m.L <= 0 || m.D <= 0 || m.r <= 0 || m.H <= 0) return PATH_ERR_INVALID_ARG;
    if (!dims_ok(m) || !wbeta_dtype_ok(dt)) return PATH_ERR_UNSUPPORTED;
    WbWs ws;
    const size_t need = carve(nullptr, m, false, ws);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    carve(workspace, m, false, ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Types t = types_of(dt);
    {
        Stage s("wbeta_gemm", st);
        const path_status ps = forward_products(x, A, Bw, u, m, t, ws, st);
        if (ps != PATH_OK) return ps;
    }
    Stage s("wbeta_fwd", st);
    const long long warps = m.BL() * m.H;
    wbeta_fwd_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(m, ws.wt, ws.ys, f, b, beta_max, w,
                                                                 t.out, beta);
    count_launches();
    return cudaGetLastError() == cudaSuccess ? PATH_OK : PATH_ERR_CUDA;
}

path_status path_wbeta_bwd(const void *x, const void *A, const void *Bw, const float *f,
                           const void *u, const float *b, float beta_max, int B, int L, int D,
                           int r, int H, int d, path_dtype dt, const void *dw, const float *dbeta,
                           void *dx, float *dA, float *dBw, float *df, float *du, float *db,
                           unsigned flags, void *workspace, size_t workspace_bytes,
                           path_stream_t stream)
{
    if (!x || !A || !Bw || !f || !u || !b || !dw || !dbeta || !dx || !dA || !dBw || !df || !du ||
        !db)
        return PATH_ERR_INVALID_ARG;
    if (!(beta_max > 0.f) || !(beta_max <= 2.f)) return PATH_ERR_INVALID_ARG;
    if (flags & ~PATH_BWD_REUSE_FWD_WORKSPACE) return PATH_ERR_INVALID_ARG;
    const Dims m{B, L, D, r, H, d};
    if (m.B <= 0 || m.L <= 0 || m.D <= 0 || m.r <= 0 || m.H <= 0) return PATH_ERR_INVALID_ARG;
    if (!dims_ok(m) || !wbeta_dtype_ok(dt)) return PATH_ERR_UNSUPPORTED;
    WbWs ws;
    const size_t need = carve(nullptr, m, true, ws);
    if (!workspace || workspace_bytes < need) return PATH_ERR_WORKSPACE;
    carve(workspace, m, true, ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Types t = types_of(dt);
    const bool tf32 = t.in != F32;
    const int ldys = m.ldys(), Hd = m.Hd();
    const int nch = nchunks(m.BL());
    if (!(flags & PATH_BWD_REUSE_FWD_WORKSPACE)) {
        Stage s("wbeta_gemm", st);
        const path_status ps = forward_products(x, A, Bw, u, m, t, ws, st);
        if (ps != PATH_OK) return ps;
    }
    {
        Stage s("wbeta_bwd", st);
        const long long warps = m.BL() * m.H;
        wbeta_dz_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(
            m, ws.wt, ws.ys, f, b, beta_max, dw, t.out, dbeta, ws.dz, ws.dys);
        conv_adjoint_kernel<<<grid_for(m.BL() * Hd), 256, 0, st>>>(m, ws.dz, f, ws.dwt);
        df_partial_kernel<<<dim3((Hd + 127) / 128, nch), 128, 0, st>>>(m, ws.dz, ws.wt, ws.dfpart);
        sum_parts_kernel<<<(Hd * 3 + 255) / 256, 256, 0, st>>>(ws.dfpart, nch, Hd * 3, df);
        colsum_partial_kernel<<<dim3((m.H + 127) / 128, nch), 128, 0, st>>>(ws.dys, m.BL(), ldys, m.r,
                                                                            m.H, ws.dbpart);
        sum_parts_kernel<<<(m.H + 255) / 256, 256, 0, st>>>(ws.dbpart, nch, m.H, db);
        count_launches(6);
        if (cudaGetLastError() != cudaSuccess) return PATH_ERR_CUDA;
    }
    Stage s("wbeta_gemm_bwd", st);
    // dBw = y^T dwt; dy = dwt Bw^T (into dys[:, :r]); d[A | U] = x^T dys; dx = dys [A | U]^T
    if (!gemm_rm(m.r, Hd, (int)m.BL(), ws.ys, ldys, true, ws.dwt, Hd, false, dBw, Hd, tf32, ws.lt, st) ||
        !gemm_rm((int)m.BL(), m.r, Hd, ws.dwt, Hd, false, ws.bw32, Hd, true, ws.dys, ldys, tf32, ws.lt, st) ||
        !gemm_rm(m.D, ldys, (int)m.BL(), ws.x32, m.D, true, ws.dys, ldys, false, ws.dwau, ldys, tf32, ws.lt,
                 st))
        return PATH_ERR_CUDA;
    float *dxf = t.out == F32 ? static_cast<float *>(dx) : ws.dx32;
    if (!gemm_rm((int)m.BL(), m.D, ldys, ws.dys, ldys, false, ws.wau, ldys, true, dxf, m.D, tf32, ws.lt,
                 st))
        return PATH_ERR_CUDA;
    if (t.out != F32)
        from_f32_kernel<<<grid_for(m.BL() * m.D), 256, 0, st>>>(ws.dx32, m.D, 0, m.BL(), m.D, dx, t.out);
    from_f32_kernel<<<grid_for((long long)m.D * m.r), 256, 0, st>>>(ws.dwau, ldys, 0, m.D, m.r, dA, F32);
    from_f32_kernel<<<grid_for((long long)m.D * m.H), 256, 0, st>>>(ws.dwau, ldys, m.r, m.D, m.H, du, F32);
    count_launches(t.out != F32 ? 3 : 2);
    return cudaGetLastError() == cudaSuccess ? PATH_OK : PATH_ERR_CUDA;
}

}  // extern "C"
