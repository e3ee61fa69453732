// Adjoint of the per-block UT transform and boundary adjustment.
//
// The forward quantities of one block of BT positions (rows of W, Q, K;
// beta; D = diag(beta)) in closed form, recomputed here for the adjoint:
//   A    = strictLower(D W W^T)          Tinv = (I + A)^{-1}      X = Tinv D
//        (X is the T^{-1} of the UT transform, Paper-Notes "训练策略")
//   What = X W                          P    = I - W^T What  (= H_e ... H_s)
//   N    = strictLower(W K^T)           U    = X N
//   Ktil = K - U^T W                    (row j: H_e ... H_{j+1} k_j)
//   M    = lower(Q W^T)                 Qtil = Q - M What   (row i: H_s ... H_i q_i)
//   Sd   = Q K^T - M U   on and below the diagonal: the full-matrix form
//          lower(QK^T) - lower(QW^T) T^{-1} strictLower(WK^T) (Paper-Notes "训练策略")
// Qtil / Ktil are the boundary-adjusted queries and keys of each block and P
// the block product (gist.science section 3, "FlashAttention-Stijl Algoritme").
#include "prep.cuh"
#include "runtime.cuh"

namespace path {

namespace {

// Tinv = (I + A)^{-1} for strictly lower A, and X = Tinv diag(beta), one block
// per CTA, by forward substitution in 16 x 16 blocks: the eight diagonal blocks
// first (their own 16-step substitutions, side by side), then block row I,
// I = 1..7: S_IJ = sum_{K=J}^{I-1} A_IK Tinv_KJ for every J < I, and
// Tinv_IJ = -Tinv_II S_IJ. Every output of a step is an independent dot
// product, so a step is one pass of the CTA.
constexpr int TB = 16, NTB = BT / TB;
__global__ void __launch_bounds__(256) tri_inverse_kernel(const float *A, float *Tinv, float *X,
                                                          const float *beta, int L, int nblk,
                                                          int batch)
{
    extern __shared__ float sm[];
    float *sA = sm;              // [BT][BT]
    float *sT = sm + BT * BT;    // [BT][BT]
    float *sS = sT + BT * BT;    // [NTB - 1][TB][TB] block sums of one block row
    for (int z = blockIdx.x; z < batch; z += gridDim.x) {
        const int h = z / nblk, blk = z % nblk;
        const long long base = (long long)z * BT * BT;
        for (int e = threadIdx.x; e < BT * BT / 4; e += blockDim.x) {
            reinterpret_cast<float4 *>(sA)[e] = reinterpret_cast<const float4 *>(A + base)[e];
            reinterpret_cast<float4 *>(sT)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        // diagonal blocks: thread (block I, column c) runs the 16-step substitution
        if (threadIdx.x < BT) {
            const int I = threadIdx.x / TB, c = threadIdx.x % TB, o = I * TB;
            float t[TB];
#pragma unroll
            for (int r = 0; r < TB; ++r) {
                float s = r == c ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < r; ++k) s = fmaf(-sA[(o + r) * BT + o + k], t[k], s);
                t[r] = r < c ? 0.f : s;
            }
#pragma unroll
            for (int r = 0; r < TB; ++r) sT[(o + r) * BT + o + c] = t[r];
        }
        __syncthreads();
        for (int I = 1; I < NTB; ++I) {
            // S_IJ[r][c] = sum_{K=J}^{I-1} sum_m A_IK[r][m] Tinv_KJ[m][c]; Tinv_KJ = 0 for K < J
            for (int e = threadIdx.x; e < I * TB * TB; e += blockDim.x) {
                const int J = e / (TB * TB), r = (e / TB) % TB, c = e % TB;
                const float *arow = sA + (I * TB + r) * BT;
                float s0 = 0.f, s1 = 0.f;
                for (int k = J * TB; k < I * TB; k += 2) {
                    s0 = fmaf(arow[k], sT[k * BT + J * TB + c], s0);
                    s1 = fmaf(arow[k + 1], sT[(k + 1) * BT + J * TB + c], s1);
                }
                sS[e] = s0 + s1;
            }
            __syncthreads();
            // Tinv_IJ = -Tinv_II S_IJ
            for (int e = threadIdx.x; e < I * TB * TB; e += blockDim.x) {
                const int J = e / (TB * TB), r = (e / TB) % TB, c = e % TB;
                const float *trow = sT + (I * TB + r) * BT + I * TB;
                const float *scol = sS + J * TB * TB + c;
                float s = 0.f;
#pragma unroll
                for (int m = 0; m < TB; ++m) s = fmaf(trow[m], scol[m * TB], s);
                sT[(I * TB + r) * BT + J * TB + c] = -s;
            }
            __syncthreads();
        }
        for (int e = threadIdx.x; e < BT * BT; e += blockDim.x) {
            const int col = e % BT;
            const int pos = blk * BT + col;
            const float b = pos < L ? beta[(long long)h * L + pos] : 0.f;
            Tinv[base + e] = sT[e];
            X[base + e] = sT[e] * b;
        }
        __syncthreads();
    }
}

// dbeta[a] = sum_{b<a} dA[a][b] G[a][b] + sum_{a'} dX[a'][a] Tinv[a'][a]
__global__ void dbeta_kernel(const float *dA, const float *G, const float *dX, const float *Tinv,
                             float *dbeta, int L, int nblk, int batch)
{
    for (int z = blockIdx.x; z < batch; z += gridDim.x) {
        const int h = z / nblk, blk = z % nblk;
        const long long base = (long long)z * BT * BT;
        const int a = threadIdx.x;
        const int pos = blk * BT + a;
        float s = 0.f;
        for (int b = 0; b < a; ++b) s = fmaf(dA[base + a * BT + b], G[base + a * BT + b], s);
        for (int r = 0; r < BT; ++r) s = fmaf(dX[base + r * BT + a], Tinv[base + r * BT + a], s);
        if (pos < L) dbeta[(long long)h * L + pos] = s;
    }
}

// out[a][b] = beta[a] * in[a][b] per block (beta = 0 past the sequence end)
__global__ void scale_rows_kernel(const float *in, float *out, const float *beta, int L, int nblk,
                                  int batch)
{
    for (int z = blockIdx.x; z < batch; z += gridDim.x) {
        const int h = z / nblk, blk = z % nblk;
        const long long base = (long long)z * BT * BT;
        for (int e = threadIdx.x; e < BT * BT; e += blockDim.x) {
            const int pos = blk * BT + e / BT;
            const float b = pos < L ? beta[(long long)h * L + pos] : 0.f;
            out[base + e] = b * in[base + e];
        }
    }
}

int grid_for(int batch) { return batch < 4096 ? batch : 4096; }

}  // namespace

cudaError_t scale_rows(const float *in, float *out, const float *beta, int L, int nblk, int batch,
                       cudaStream_t st)
{
    scale_rows_kernel<<<grid_for(batch), 256, 0, st>>>(in, out, beta, L, nblk, batch);
    count_launches();
    return cudaGetLastError();
}

// --- operand builders -------------------------------------------------------
static Operand user_rows(const void *p, int dt, int L, int d)  // [nh, L, d] user tensor
{
    Operand o;
    o.p = p;
    o.dt = dt;
    o.sh = (long long)L * d;
    o.sb = (long long)BT * d;
    o.ld = d;
    o.seq = L;
    return o;
}

static Operand padded_rows(const void *p, int dt, int Lp, int d)  // [nh, Lp, d] workspace
{
    Operand o;
    o.p = p;
    o.dt = dt;
    o.sh = (long long)Lp * d;
    o.sb = (long long)BT * d;
    o.ld = d;
    return o;
}

static Operand blk_mat(const void *p, int dt, int nblk, int rows, int cols)  // [nh, nblk, rows, cols]
{
    Operand o;
    o.p = p;
    o.dt = dt;
    o.sh = (long long)nblk * rows * cols;
    o.sb = (long long)rows * cols;
    o.ld = cols;
    return o;
}

static Operand T_(Operand o)
{
    o.trans = 1;
    return o;
}

static Operand masked(Operand o, int m)
{
    o.mask = m;
    return o;
}

static void set_out(GemmArgs &g, void *p, int dt, long long sh, long long sb, int ldc, int c_seq)
{
    g.c = p;
    g.cdt = dt;
    g.csh = sh;
    g.csb = sb;
    g.ldc = ldc;
    g.c_seq = c_seq;
}

static GemmArgs base_args(const PrepDims &D, int M, int N, int K)
{
    GemmArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.nblk = D.nblk;
    g.batch = D.nh * D.nblk;
    return g;
}

static void term(GemmArgs &g, Operand a, Operand b, float alpha)
{
    g.t[g.nterms].a = a;
    g.t[g.nterms].b = b;
    g.t[g.nterms].alpha = alpha;
    ++g.nterms;
}

static void out_blk(GemmArgs &g, const PrepDims &D, float *p, int rows, int cols, int outmask = 0)
{
    set_out(g, p, F32, (long long)D.nblk * rows * cols, (long long)rows * cols, cols, -1);
    g.outmask = outmask;
}

#define CK(x)                                 \
    do {                                      \
        cudaError_t e_ = (x);                 \
        if (e_ != cudaSuccess) return e_;     \
    } while (0)

// bf16 / fp16 inputs: the products on the tensor cores in TF32; fp32 inputs: fp32
// on CUDA cores (the fp32 mode's precision)
static cudaError_t gemm(const PrepDims &D, GemmArgs g, const PrepScratch &s, cudaStream_t st)
{
    g.err = s.err;
    if (D.dt != F32 && gemm_tc_supported(g)) return gemm_batched_tc(g, st);
    return gemm_batched(g, st);
}

size_t prep_scratch_bytes(const PrepDims &D, bool backward)
{
    Carver c(nullptr);
    PrepScratch s;
    carve_prep_scratch(c, D, backward, s);
    return c.bytes();
}

void carve_prep_scratch(Carver &c, const PrepDims &D, bool backward, PrepScratch &s)
{
    const size_t nb = (size_t)D.nh * D.nblk;
    const size_t sq = nb * BT * BT, rd = nb * BT * D.d;
    s.G = c.take<float>(sq);
    s.A = c.take<float>(sq);
    s.Tinv = c.take<float>(sq);
    s.X = c.take<float>(sq);
    s.N = c.take<float>(sq);
    s.U = c.take<float>(sq);
    s.M = c.take<float>(sq);
    s.What = c.take<float>(rd);
    if (backward) {
        s.dM = c.take<float>(sq);
        s.dU = c.take<float>(sq);
        s.dN = c.take<float>(sq);
        s.dX = c.take<float>(sq);
        s.tmp = c.take<float>(sq);
        s.dA = c.take<float>(sq);
        s.dG = c.take<float>(sq);
        s.dWhat = c.take<float>(rd);
        s.dWacc = c.take<float>(rd);
    }
}

void carve_ut_save(Carver &c, const PrepDims &D, UtSave &s)
{
    const size_t nb = (size_t)D.nh * D.nblk, d = D.d, hb = BT / 2;
    s.What = c.take<f16>(nb * 2 * hb * d);
    s.U = c.take<f16>(nb * 2 * hb * hb);
    s.X = c.take<f16>(nb * 2 * hb * hb);
    s.M = c.take<f16>(nb * 2 * hb * hb);
    s.Kta = c.take<f16>(nb * hb * d);
    s.Qtb = c.take<f16>(nb * hb * d);
    s.Pa = c.take<f16>(nb * d * d);
    s.Pb = c.take<f16>(nb * d * d);
    s.dP = d == 128 ? c.take<f16>(nb * 2 * d * d) : nullptr;
}

// Closed-form forward quantities the adjoint needs: A, G, Tinv, X, What, N, U, M.
static cudaError_t prep_core(const PrepDims &D, const PrepInputs &in, const PrepScratch &s,
                             cudaStream_t st)
{
    const int L = D.L, d = D.d, nb = D.nblk;
    const Operand W = user_rows(in.w, D.dt, L, d), K = user_rows(in.k, D.dt, L, d),
                  Q = user_rows(in.q, D.dt, L, d);
    {   // G = W W^T ; A = strictLower(D G)
        GemmArgs g = base_args(D, BT, BT, d);
        term(g, W, T_(W), 1.f);
        out_blk(g, D, s.G, BT, BT);
        CK(gemm(D, g, s, st));
        g.rowscale = in.beta;
        g.rs_sh = L;
        g.rs_sb = BT;
        g.rs_seq = L;
        out_blk(g, D, s.A, BT, BT, MASK_STRICT_LOWER);
        CK(gemm(D, g, s, st));
    }
    {
        const int batch = D.nh * nb;
        const size_t smem = (2 * BT * BT + (NTB - 1) * TB * TB) * sizeof(float);
        CK(cudaFuncSetAttribute(tri_inverse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
        tri_inverse_kernel<<<grid_for(batch), 256, smem, st>>>(s.A, s.Tinv, s.X, in.beta, L, nb,
                                                               batch);
        count_launches();
        CK(cudaGetLastError());
    }
    const Operand X = blk_mat(s.X, F32, nb, BT, BT);
    {   // What = X W
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, X, W, 1.f);
        out_blk(g, D, s.What, BT, d);
        CK(gemm(D, g, s, st));
    }
    {   // N = strictLower(W K^T)
        GemmArgs g = base_args(D, BT, BT, d);
        term(g, W, T_(K), 1.f);
        out_blk(g, D, s.N, BT, BT, MASK_STRICT_LOWER);
        CK(gemm(D, g, s, st));
    }
    {   // U = X N
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, X, blk_mat(s.N, F32, nb, BT, BT), 1.f);
        out_blk(g, D, s.U, BT, BT);
        CK(gemm(D, g, s, st));
    }
    {   // M = lower(Q W^T)
        GemmArgs g = base_args(D, BT, BT, d);
        term(g, Q, T_(W), 1.f);
        out_blk(g, D, s.M, BT, BT, MASK_LOWER);
        CK(gemm(D, g, s, st));
    }
    return cudaSuccess;
}

cudaError_t prep_forward_gemm(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                              const PrepScratch &s, cudaStream_t st)
{
    CK(prep_core(D, in, s, st));
    const int L = D.L, d = D.d, nb = D.nblk, Lp = nb * BT;
    const Operand W = user_rows(in.w, D.dt, L, d), K = user_rows(in.k, D.dt, L, d),
                  Q = user_rows(in.q, D.dt, L, d);
    const Operand U = blk_mat(s.U, F32, nb, BT, BT), M = blk_mat(s.M, F32, nb, BT, BT),
                  What = blk_mat(s.What, F32, nb, BT, d);
    {   // P = I - W^T What
        GemmArgs g = base_args(D, d, d, BT);
        term(g, T_(W), What, -1.f);
        g.add_identity = 1;
        set_out(g, out.Pm, out.tdt, (long long)nb * d * d, (long long)d * d, d, -1);
        CK(gemm(D, g, s, st));
    }
    {   // Qtil = Q - M What (rows past L: zero)
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, M, What, -1.f);
        g.addend = Q;
        g.gamma = 1.f;
        set_out(g, out.Qt, out.tdt, (long long)Lp * d, (long long)BT * d, d, -1);
        CK(gemm(D, g, s, st));
    }
    {   // Ktil = K - U^T W
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, T_(U), W, -1.f);
        g.addend = K;
        g.gamma = 1.f;
        set_out(g, out.Kt, out.tdt, (long long)Lp * d, (long long)BT * d, d, -1);
        CK(gemm(D, g, s, st));
    }
    {   // Sd = lower(Q K^T - M U)
        GemmArgs g = base_args(D, BT, BT, d);
        term(g, Q, T_(K), 1.f);
        out_blk(g, D, out.Sd, BT, BT);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, BT, BT);
        term(g2, M, U, -1.f);
        g2.addend = blk_mat(out.Sd, F32, nb, BT, BT);
        g2.gamma = 1.f;
        out_blk(g2, D, out.Sd, BT, BT, MASK_LOWER);
        CK(gemm(D, g2, s, st));
    }
    return cudaSuccess;
}

cudaError_t prep_backward(const PrepDims &D, const PrepInputs &in, const PrepScratch &s,
                          const PrepGrads &gr, cudaStream_t st)
{
    CK(prep_core(D, in, s, st));
    const int L = D.L, d = D.d, nb = D.nblk, Lp = nb * BT;
    const Operand W = user_rows(in.w, D.dt, L, d), K = user_rows(in.k, D.dt, L, d),
                  Q = user_rows(in.q, D.dt, L, d);
    const Operand U = blk_mat(s.U, F32, nb, BT, BT), M = blk_mat(s.M, F32, nb, BT, BT),
                  What = blk_mat(s.What, F32, nb, BT, d), X = blk_mat(s.X, F32, nb, BT, BT),
                  Nm = blk_mat(s.N, F32, nb, BT, BT), Tinv = blk_mat(s.Tinv, F32, nb, BT, BT),
                  G = blk_mat(s.G, F32, nb, BT, BT);
    const Operand dSl = masked(blk_mat(gr.dSd, F32, nb, BT, BT), MASK_LOWER);
    const Operand dQt = padded_rows(gr.dQt, F32, Lp, d), dKt = padded_rows(gr.dKt, F32, Lp, d);
    const Operand dP = blk_mat(gr.dPm, F32, nb, d, d);
    const Operand dM = blk_mat(s.dM, F32, nb, BT, BT), dU = blk_mat(s.dU, F32, nb, BT, BT),
                  dN = blk_mat(s.dN, F32, nb, BT, BT), dX = blk_mat(s.dX, F32, nb, BT, BT),
                  tmp = blk_mat(s.tmp, F32, nb, BT, BT), dA = blk_mat(s.dA, F32, nb, BT, BT),
                  dGm = blk_mat(s.dG, F32, nb, BT, BT), dWhat = blk_mat(s.dWhat, F32, nb, BT, d),
                  dWacc = blk_mat(s.dWacc, F32, nb, BT, d);
    const long long ush = (long long)L * d, usb = (long long)BT * d;
    {   // dM = lower(-dSl U^T - dQt What^T)
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, dSl, T_(U), -1.f);
        out_blk(g, D, s.dM, BT, BT, MASK_LOWER);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, BT, d);
        term(g2, dQt, T_(What), -1.f);
        g2.addend = dM;
        g2.gamma = 1.f;
        out_blk(g2, D, s.dM, BT, BT, MASK_LOWER);
        CK(gemm(D, g2, s, st));
    }
    {   // dq = dQt + dSl K + dM W
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, dSl, K, 1.f);
        term(g, dM, W, 1.f);
        g.addend = dQt;
        g.gamma = 1.f;
        set_out(g, gr.dq, D.odt, ush, usb, d, L);
        CK(gemm(D, g, s, st));
    }
    {   // dU = -M^T dSl - W dKt^T
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, T_(M), dSl, -1.f);
        out_blk(g, D, s.dU, BT, BT);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, BT, d);
        term(g2, W, T_(dKt), -1.f);
        g2.addend = dU;
        g2.gamma = 1.f;
        out_blk(g2, D, s.dU, BT, BT);
        CK(gemm(D, g2, s, st));
    }
    {   // dN = strictLower(X^T dU)
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, T_(X), dU, 1.f);
        out_blk(g, D, s.dN, BT, BT, MASK_STRICT_LOWER);
        CK(gemm(D, g, s, st));
    }
    {   // dk = dKt + dSl^T Q + dN^T W
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, T_(dSl), Q, 1.f);
        term(g, T_(dN), W, 1.f);
        g.addend = dKt;
        g.gamma = 1.f;
        set_out(g, gr.dk, D.odt, ush, usb, d, L);
        CK(gemm(D, g, s, st));
    }
    {   // dWhat = -M^T dQt - W dP
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, T_(M), dQt, -1.f);
        out_blk(g, D, s.dWhat, BT, d);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, d, d);
        term(g2, W, dP, -1.f);
        g2.addend = dWhat;
        g2.gamma = 1.f;
        out_blk(g2, D, s.dWhat, BT, d);
        CK(gemm(D, g2, s, st));
    }
    {   // dX = dU N^T + dWhat W^T
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, dU, T_(Nm), 1.f);
        out_blk(g, D, s.dX, BT, BT);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, BT, d);
        term(g2, dWhat, T_(W), 1.f);
        g2.addend = dX;
        g2.gamma = 1.f;
        out_blk(g2, D, s.dX, BT, BT);
        CK(gemm(D, g2, s, st));
    }
    {   // dA = strictLower(-(Tinv^T dX) X^T)   (adjoint of Tinv = (I + A)^{-1}, X = Tinv D)
        GemmArgs g = base_args(D, BT, BT, BT);
        term(g, T_(Tinv), dX, 1.f);
        out_blk(g, D, s.tmp, BT, BT);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, BT, BT);
        term(g2, tmp, T_(X), -1.f);
        out_blk(g2, D, s.dA, BT, BT, MASK_STRICT_LOWER);
        CK(gemm(D, g2, s, st));
    }
    // dG = strictLower(D dA): dA is strictly lower already, scale its rows by beta
    CK(scale_rows(s.dA, s.dG, in.beta, L, nb, D.nh * nb, st));
    {
        const int batch = D.nh * nb;
        dbeta_kernel<<<grid_for(batch), BT, 0, st>>>(s.dA, s.G, s.dX, s.Tinv, gr.dbeta, L, nb,
                                                     batch);
        count_launches();
        CK(cudaGetLastError());
    }
    {   // dW = -U dKt + dN K + dM^T Q - What dP^T + X^T dWhat + (dG + dG^T) W
        GemmArgs g = base_args(D, BT, d, BT);
        term(g, U, dKt, -1.f);
        term(g, dN, K, 1.f);
        term(g, T_(dM), Q, 1.f);
        out_blk(g, D, s.dWacc, BT, d);
        CK(gemm(D, g, s, st));
        GemmArgs g2 = base_args(D, BT, d, d);
        term(g2, What, T_(dP), -1.f);
        g2.addend = dWacc;
        g2.gamma = 1.f;
        out_blk(g2, D, s.dWacc, BT, d);
        CK(gemm(D, g2, s, st));
        GemmArgs g3 = base_args(D, BT, d, BT);
        term(g3, T_(X), dWhat, 1.f);
        term(g3, dGm, W, 1.f);
        term(g3, T_(dGm), W, 1.f);
        g3.addend = dWacc;
        g3.gamma = 1.f;
        set_out(g3, gr.dw, D.odt, ush, usb, d, L);
        CK(gemm(D, g3, s, st));
    }
    return cudaSuccess;
}

}  // namespace path
