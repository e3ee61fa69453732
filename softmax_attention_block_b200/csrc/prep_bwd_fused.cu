// Adjoint of the per-block prep, head dim 64, fused per block (fp32).
//
// The attention backward hands over, per 128-position block, the adjoints of
// the boundary-adjusted queries/keys (dQtil, dKtil), of the block product
// (dP) and of the diagonal-block logits (dSd). They are carried to dq, dk, dw
// and dbeta in two kernels:
//
// 1. compose_adj: a 128-block is two 64-position halves a (first) and b. With
//    the halves' own boundary-adjusted queries/keys and products,
//      Qtil[b] = Qtil_b P_a,  Ktil[a] = Ktil_a P_b^T,  P = P_b P_a,
//      Sd[b, a] = Qtil_b Ktil_a^T     (Sd[a, a], Sd[b, b] are the halves' own),
//    so the 128-level adjoints become per-half ones by a few 64x64 products.
//    The halves' quantities are recomputed by the same rank-one recurrences
//    as the forward prep (64 steps).
// 2. ut_adj64: per 64-position half, the UT transform in closed form
//    (Paper-Notes "训练策略": T^{-1} = (I + strictLower(D W W^T))^{-1} D):
//      A = strictLower(D W W^T), N = strictLower(W K^T), M = lower(Q W^T),
//      [What | U] = (I + A)^{-1} D [W | N]           (one triangular solve)
//      Qtil = Q - M What, Ktil = K - U^T W, P = I - W^T What, Sd = Q K^T - M U,
//    and its adjoint, where (I + A)^{-T} applied to [dWhat | dU] gives dR and
//    dA = strictLower(-dR [What | U]^T), so T^{-1} itself is never formed.
#include "prep.cuh"
#include "runtime.cuh"

namespace path {

namespace {

constexpr int HB = 64;       // half block
constexpr int D = 64;        // head dim of this path
constexpr int LD = HB + 1;   // padded row stride of the 64x64 shared matrices
constexpr int NT = 256;

enum { OUT_ALL = 0, OUT_LOWER = 1, OUT_STRICT = 2 };

// C (64x64, stride LD, shared) (=|+=) alpha * op(A) op(B), op = transpose if TA/TB.
// A, B: 64x64 with row stride lda/ldb, in shared or global memory, element
// types AT/BT; rows of a non-transposed B at or past b_rows read as zero (and
// are never loaded). 256 threads, 4x4 outputs each. Ends with a barrier.
template <bool TA, bool TB, typename AT, typename BT>
__device__ void bgemm(float *C, const AT *A, int lda, const BT *B, int ldb, float alpha,
                      bool accumulate, int mask, int b_rows = HB)
{
    const int t = threadIdx.x;
    const int i0 = (t >> 4) * 4, j0 = (t & 15) * 4;
    float acc[4][4] = {};
#pragma unroll 4
    for (int k = 0; k < HB; ++k) {
        float a[4], b[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) a[r] = to_f(TA ? A[k * lda + i0 + r] : A[(i0 + r) * lda + k]);
#pragma unroll
        for (int c = 0; c < 4; ++c)  // a non-transposed B reads row k only below b_rows
            b[c] = TB ? to_f(B[(j0 + c) * ldb + k]) : (k < b_rows ? to_f(B[k * ldb + j0 + c]) : 0.f);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();  // C may alias an operand of an earlier phase, never of this one
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = i0 + r, j = j0 + c;
            float v = alpha * acc[r][c] + (accumulate ? C[i * LD + j] : 0.f);
            if ((mask == OUT_LOWER && j > i) || (mask == OUT_STRICT && j >= i)) v = 0.f;
            C[i * LD + j] = v;
        }
    __syncthreads();
}

// Row-scale and mask in place: X[i][j] *= s[i] (masked entries zeroed).
__device__ void scale_rows_mask(float *X, const float *s, int mask)
{
    for (int e = threadIdx.x; e < HB * HB; e += NT) {
        const int i = e / HB, j = e % HB;
        float v = X[i * LD + j] * s[i];
        if ((mask == OUT_LOWER && j > i) || (mask == OUT_STRICT && j >= i)) v = 0.f;
        X[i * LD + j] = v;
    }
    __syncthreads();
}

template <typename T>
__device__ void load_rows(float *dst, const T *src, int nvalid)  // 64 rows x 64 (stride 64)
{
    for (int e = threadIdx.x; e < HB * D; e += NT) {
        const int r = e / D, c = e % D;
        dst[r * LD + c] = r < nvalid ? to_f(src[(long long)r * D + c]) : 0.f;
    }
}

__device__ void load_f32(float *dst, const float *src, int ld_src)
{
    for (int e = threadIdx.x; e < HB * HB; e += NT) {
        const int r = e / HB, c = e % HB;
        dst[r * LD + c] = src[(long long)r * ld_src + c];
    }
}

// x <- H_t x = x - beta_t w_t (w_t . x), with w_t a row of the shared W (stride LD)
__device__ __forceinline__ void apply_h(float *x, const float *sW, const float *sB, int t)
{
    const float *wt = sW + t * LD;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int c = 0; c < D; c += 2) {
        a0 = fmaf(wt[c], x[c], a0);
        a1 = fmaf(wt[c + 1], x[c + 1], a1);
    }
    const float coef = sB[t] * (a0 + a1);
#pragma unroll
    for (int c = 0; c < D; ++c) x[c] = fmaf(-coef, wt[c], x[c]);
}

// ---------------------------------------------------------------------------
// 1. 128-level adjoints -> per-half adjoints (in place for dQt / dKt)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(NT) compose_adj_kernel(const T *q, const T *k, const T *w,
                                                         const float *beta, int L, int nblk,
                                                         float *dQt, float *dKt, const float *dPm,
                                                         const float *dSd, float *dP64)
{
    extern __shared__ float sm[];
    float *sW = sm;                   // [128][LD]
    float *sBt = sW + BT * LD;        // [128]
    float *sKa = sBt + BT;            // Ktil_a [64][LD]
    float *sQb = sKa + HB * LD;       // Qtil_b
    float *sPa = sQb + HB * LD;       // P_a
    float *sPb = sPa + HB * LD;       // P_b
    float *sDX = sPb + HB * LD;       // dSd[b, a]
    float *sDQb = sDX + HB * LD;      // dQtil[b]
    float *sDKa = sDQb + HB * LD;     // dKtil[a]
    float *sDP = sDKa + HB * LD;      // dP
    float *sOut = sDP + HB * LD;      // product staging
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int Lp = nblk * BT;
    const long long row0 = (long long)h * L + (long long)J * BT;
    const int nvalid = min(BT, L - J * BT);
    for (int e = tid; e < BT * D; e += NT) {
        const int r = e / D, c = e % D;
        sW[r * LD + c] = r < nvalid ? to_f(w[(row0 + r) * D + c]) : 0.f;
    }
    for (int r = tid; r < BT; r += NT) sBt[r] = r < nvalid ? beta[row0 + r] : 0.f;
    const float *dsd = dSd + ((long long)h * nblk + J) * BT * BT;
    const long long prow = (long long)h * Lp + (long long)J * BT;
    for (int e = tid; e < HB * HB; e += NT) {
        const int r = e / HB, c = e % HB;
        sDX[r * LD + c] = dsd[(long long)(HB + r) * BT + c];
        sDQb[r * LD + c] = dQt[(prow + HB + r) * D + c];
        sDKa[r * LD + c] = dKt[(prow + r) * D + c];
        sDP[r * LD + c] = dPm[((long long)h * nblk + J) * D * D + r * D + c];
    }
    __syncthreads();
    // the halves' own quantities, by recurrence
    {
        float x[D];
        const int g = tid / HB, r = tid % HB;
        if (g == 0) {  // key r of half a carried to the end of half a
            for (int c = 0; c < D; ++c) x[c] = r < nvalid ? to_f(k[(row0 + r) * D + c]) : 0.f;
            for (int t = r + 1; t < HB; ++t) apply_h(x, sW, sBt, t);
            for (int c = 0; c < D; ++c) sKa[r * LD + c] = x[c];
        } else if (g == 1) {  // query 64+r of half b carried back to the start of half b
            const int i = HB + r;
            for (int c = 0; c < D; ++c) x[c] = i < nvalid ? to_f(q[(row0 + i) * D + c]) : 0.f;
            for (int t = i; t >= HB; --t) apply_h(x, sW, sBt, t);
            for (int c = 0; c < D; ++c) sQb[r * LD + c] = x[c];
        } else {  // column r of P_a (g == 2) or P_b (g == 3)
            const int t0 = g == 2 ? 0 : HB;
            for (int c = 0; c < D; ++c) x[c] = c == r ? 1.f : 0.f;
            for (int t = t0; t < t0 + HB; ++t) apply_h(x, sW, sBt, t);
            float *dst = g == 2 ? sPa : sPb;
            for (int c = 0; c < D; ++c) dst[c * LD + r] = x[c];
        }
    }
    __syncthreads();
    auto store = [&](float *dst, long long ld) {
        for (int e = tid; e < HB * HB; e += NT) {
            const int r = e / HB, c = e % HB;
            dst[(long long)r * ld + c] = sOut[r * LD + c];
        }
        __syncthreads();
    };
    // dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a
    bgemm<false, true>(sOut, sDQb, LD, sPa, LD, 1.f, false, OUT_ALL);
    bgemm<false, false>(sOut, sDX, LD, sKa, LD, 1.f, true, OUT_ALL);
    store(dQt + (prow + HB) * D, D);
    // dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b
    bgemm<false, false>(sOut, sDKa, LD, sPb, LD, 1.f, false, OUT_ALL);
    bgemm<true, false>(sOut, sDX, LD, sQb, LD, 1.f, true, OUT_ALL);
    store(dKt + prow * D, D);
    // dP_a = Qtil_b^T dQtil[b] + P_b^T dP
    bgemm<true, false>(sOut, sQb, LD, sDQb, LD, 1.f, false, OUT_ALL);
    bgemm<true, false>(sOut, sPb, LD, sDP, LD, 1.f, true, OUT_ALL);
    store(dP64 + ((long long)h * 2 * nblk + 2 * J) * D * D, D);
    // dP_b = dKtil[a]^T Ktil_a + dP P_a^T
    bgemm<true, false>(sOut, sDKa, LD, sKa, LD, 1.f, false, OUT_ALL);
    bgemm<false, true>(sOut, sDP, LD, sPa, LD, 1.f, true, OUT_ALL);
    store(dP64 + ((long long)h * 2 * nblk + 2 * J + 1) * D * D, D);
}

// ---------------------------------------------------------------------------
// 2. UT adjoint of one 64-position half
// ---------------------------------------------------------------------------
template <typename T, typename TO>
__global__ void __launch_bounds__(NT) ut_adj64_kernel(const T *q, const T *k, const T *w,
                                                      const float *beta, int L, int nblk,
                                                      const float *dQt, const float *dKt,
                                                      const float *dP64, const float *dSd,
                                                      TO *dq, TO *dk, TO *dw, float *dbeta)
{
    extern __shared__ float sm[];
    float *sW = sm, *sQ = sW + HB * LD, *sA = sQ + HB * LD, *sN = sA + HB * LD,
          *sM = sN + HB * LD, *sWh = sM + HB * LD, *sU = sWh + HB * LD, *sDQ = sU + HB * LD,
          *sDK = sDQ + HB * LD, *sDP = sDK + HB * LD, *sDS = sDP + HB * LD,
          *sDWh = sDS + HB * LD, *sDU = sDWh + HB * LD, *sB = sDU + HB * LD,
          *sRed = sB + HB;  // [2][128] partial sums of the solves
    const int blk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int J = blk / 2, half = blk % 2;
    const int Lp = nblk * BT;
    const int pos0 = J * BT + half * HB;
    const int nvalid = max(0, min(HB, L - pos0));
    const long long row0 = (long long)h * L + pos0;
    const T *Kg = k + row0 * D;  // read only below nvalid rows
    load_rows(sW, w + row0 * D, nvalid);
    load_rows(sQ, q + row0 * D, nvalid);
    for (int r = tid; r < HB; r += NT) sB[r] = r < nvalid ? beta[row0 + r] : 0.f;
    const long long prow = (long long)h * Lp + pos0;
    load_f32(sDQ, dQt + prow * D, D);
    load_f32(sDK, dKt + prow * D, D);
    load_f32(sDP, dP64 + ((long long)h * 2 * nblk + blk) * D * D, D);
    load_f32(sDS, dSd + ((long long)h * nblk + J) * BT * BT + (long long)(half * HB) * BT + half * HB, BT);
    // K of this half (zero past the end) staged in sWh until the solve overwrites it
    load_rows(sWh, Kg, nvalid);
    __syncthreads();
    // forward quantities
    bgemm<false, true>(sA, sW, LD, sW, LD, 1.f, false, OUT_STRICT);   // W W^T
    scale_rows_mask(sA, sB, OUT_STRICT);                                // A = strictLower(D W W^T)
    bgemm<false, true>(sN, sW, LD, sWh, LD, 1.f, false, OUT_STRICT);  // N = strictLower(W K^T)
    bgemm<false, true>(sM, sQ, LD, sW, LD, 1.f, false, OUT_LOWER);    // M = lower(Q W^T)
    // [What | U] = (I + A)^{-1} D [W | N]: forward substitution, 128 right-hand sides
    for (int e = tid; e < HB * HB; e += NT) {
        const int r = e / HB, c = e % HB;
        sWh[r * LD + c] = sB[r] * sW[r * LD + c];
        sU[r * LD + c] = sB[r] * sN[r * LD + c];
    }
    __syncthreads();
    {
        const int col = tid % 128, part = tid / 128;  // two threads per right-hand side
        float *Z = col < HB ? sWh : sU;
        const int c = col % HB;
        for (int i = 1; i < HB; ++i) {
            const int mid = i / 2;
            const int k0 = part == 0 ? 0 : mid, k1 = part == 0 ? mid : i;
            float s = 0.f;
            for (int kk = k0; kk < k1; ++kk) s = fmaf(sA[i * LD + kk], Z[kk * LD + c], s);
            sRed[part * 128 + col] = s;
            __syncthreads();
            if (part == 0) Z[i * LD + c] -= sRed[col] + sRed[128 + col];
            __syncthreads();
        }
    }
    // adjoint
    bgemm<true, false>(sDWh, sM, LD, sDQ, LD, -1.f, false, OUT_ALL);   // -M^T dQtil
    bgemm<false, false>(sDWh, sW, LD, sDP, LD, -1.f, true, OUT_ALL);   // -W dP
    bgemm<false, true>(sDU, sW, LD, sDK, LD, -1.f, false, OUT_ALL);    // -W dKtil^T
    bgemm<true, false>(sDU, sM, LD, sDS, LD, -1.f, true, OUT_ALL);     // -M^T dSd
    bgemm<false, true>(sM, sDQ, LD, sWh, LD, -1.f, false, OUT_LOWER);  // dM (over M)
    bgemm<false, true>(sM, sDS, LD, sU, LD, -1.f, true, OUT_LOWER);
    // dq = dQtil + dSd K + dM W
    {
        bgemm<false, false>(sDQ, sDS, LD, Kg, D, 1.f, true, OUT_ALL, nvalid);
        bgemm<false, false>(sDQ, sM, LD, sW, LD, 1.f, true, OUT_ALL);
        for (int e = tid; e < HB * D; e += NT) {
            const int r = e / D, c = e % D;
            if (r < nvalid) dq[(row0 + r) * D + c] = from_f<TO>(sDQ[r * LD + c]);
        }
        __syncthreads();
    }
    // dR = (I + A)^{-T} [dWhat | dU]: backward substitution
    {
        const int col = tid % 128, part = tid / 128;
        float *Z = col < HB ? sDWh : sDU;
        const int c = col % HB;
        for (int i = HB - 2; i >= 0; --i) {
            const int n = HB - 1 - i, mid = i + 1 + n / 2;
            const int k0 = part == 0 ? i + 1 : mid, k1 = part == 0 ? mid : HB;
            float s = 0.f;
            for (int kk = k0; kk < k1; ++kk) s = fmaf(sA[kk * LD + i], Z[kk * LD + c], s);
            sRed[part * 128 + col] = s;
            __syncthreads();
            if (part == 0) Z[i * LD + c] -= sRed[col] + sRed[128 + col];
            __syncthreads();
        }
    }
    // dA = strictLower(-(dR_w What^T + dR_n U^T))   (into sDQ, free now)
    bgemm<false, true>(sDQ, sDWh, LD, sWh, LD, -1.f, false, OUT_STRICT);
    bgemm<false, true>(sDQ, sDU, LD, sU, LD, -1.f, true, OUT_STRICT);
    // dbeta_a = dR_w[a].W[a] + dR_n[a].N[a] + sum_{b<a} dA[a][b] (W[a].W[b])
    if (tid < HB) {
        const int a = tid;
        float s = 0.f;
        for (int c = 0; c < D; ++c) s = fmaf(sDWh[a * LD + c], sW[a * LD + c], s);
        for (int c = 0; c < HB; ++c) s = fmaf(sDU[a * LD + c], sN[a * LD + c], s);
        for (int b = 0; b < a; ++b) {
            float g = 0.f;
            for (int c = 0; c < D; ++c) g = fmaf(sW[a * LD + c], sW[b * LD + c], g);
            s = fmaf(sDQ[a * LD + b], g, s);
        }
        if (a < nvalid) dbeta[row0 + a] = s;
    }
    __syncthreads();
    // dN = strictLower(D dR_n) (over dR_n); dG = strictLower(D dA) (over dA)
    scale_rows_mask(sDU, sB, OUT_STRICT);
    // dk = dKtil + dSd^T Q + dN^T W      (into sA, free after the solves)
    for (int e = tid; e < HB * HB; e += NT) sA[(e / HB) * LD + e % HB] = sDK[(e / HB) * LD + e % HB];
    __syncthreads();
    bgemm<true, false>(sA, sDS, LD, sQ, LD, 1.f, true, OUT_ALL);
    bgemm<true, false>(sA, sDU, LD, sW, LD, 1.f, true, OUT_ALL);
    for (int e = tid; e < HB * D; e += NT) {
        const int r = e / D, c = e % D;
        if (r < nvalid) dk[(row0 + r) * D + c] = from_f<TO>(sA[r * LD + c]);
    }
    __syncthreads();
    scale_rows_mask(sDQ, sB, OUT_STRICT);  // dG
    // dw = -U dKtil - What dP^T + dM^T Q + D dR_w + dN K + (dG + dG^T) W   (into sA)
    for (int e = tid; e < HB * HB; e += NT) {
        const int r = e / HB, c = e % HB;
        sA[r * LD + c] = sB[r] * sDWh[r * LD + c];
    }
    __syncthreads();
    bgemm<false, false>(sA, sU, LD, sDK, LD, -1.f, true, OUT_ALL);
    bgemm<false, true>(sA, sWh, LD, sDP, LD, -1.f, true, OUT_ALL);
    bgemm<true, false>(sA, sM, LD, sQ, LD, 1.f, true, OUT_ALL);
    bgemm<false, false>(sA, sDU, LD, Kg, D, 1.f, true, OUT_ALL, nvalid);
    bgemm<false, false>(sA, sDQ, LD, sW, LD, 1.f, true, OUT_ALL);
    bgemm<true, false>(sA, sDQ, LD, sW, LD, 1.f, true, OUT_ALL);
    for (int e = tid; e < HB * D; e += NT) {
        const int r = e / D, c = e % D;
        if (r < nvalid) dw[(row0 + r) * D + c] = from_f<TO>(sA[r * LD + c]);
    }
}

template <typename T, typename TO>
cudaError_t run(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g, float *dP64,
                cudaStream_t st)
{
    const size_t smc = (BT * LD + BT + 9 * HB * LD) * sizeof(float);
    const size_t smu = (13 * HB * LD + HB + 256) * sizeof(float);
    auto kc = compose_adj_kernel<T>;
    auto ku = ut_adj64_kernel<T, TO>;
    cudaError_t e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ku, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smu);
    if (e != cudaSuccess) return e;
    const T *q = static_cast<const T *>(in.q), *k = static_cast<const T *>(in.k),
            *w = static_cast<const T *>(in.w);
    kc<<<dim3(Dm.nblk, Dm.nh), NT, smc, st>>>(q, k, w, in.beta, Dm.L, Dm.nblk,
                                              const_cast<float *>(g.dQt), const_cast<float *>(g.dKt),
                                              g.dPm, g.dSd, dP64);
    count_launches();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ku<<<dim3(2 * Dm.nblk, Dm.nh), NT, smu, st>>>(q, k, w, in.beta, Dm.L, Dm.nblk, g.dQt, g.dKt,
                                                  dP64, g.dSd, static_cast<TO *>(g.dq),
                                                  static_cast<TO *>(g.dk), static_cast<TO *>(g.dw),
                                                  g.dbeta);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool prep_backward_fused_supported(const PrepDims &Dm) { return Dm.d == D; }

// dQt and dKt are overwritten (used as scratch for the per-half adjoints).
cudaError_t prep_backward_fused(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g,
                                float *dP64, cudaStream_t st)
{
    if (Dm.dt == F32) return run<float, float>(Dm, in, g, dP64, st);
    if (Dm.odt == BF16) return run<bf16, bf16>(Dm, in, g, dP64, st);
    return run<bf16, float>(Dm, in, g, dP64, st);
}

}  // namespace path
