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
#include <type_traits>

#include "prep.cuh"
#include "runtime.cuh"
#include "ut64.cuh"

namespace path {

namespace {

using namespace ut64;

constexpr int WLD = D + 4;  // row stride of the recurrences' W (halves 4 floats apart)

// Column c of a row of the recurrences' W: the two 32-column halves sit 36
// floats apart, so the two lanes of a row read different banks.
__device__ __forceinline__ int wx(int t, int c) { return t * WLD + c + (c >= 32 ? 4 : 0); }

// x <- H_t x = x - beta_t w_t (w_t . x) on this lane's 32 columns (half p of
// the row; the partner lane holds the other half), or x unchanged when !on.
// Every lane of the warp calls it with the same t (it shuffles).
__device__ __forceinline__ void apply_h_half(float (&x)[32], const float *sW, const float *sB, int t,
                                             int p, bool on = true)
{
    const float4 *wt = reinterpret_cast<const float4 *>(sW + wx(t, 32 * p));
    float w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 v = wt[c];
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
        a0 = fmaf(w[c], x[c], a0);
        a1 = fmaf(w[c + 1], x[c + 1], a1);
        a2 = fmaf(w[c + 2], x[c + 2], a2);
        a3 = fmaf(w[c + 3], x[c + 3], a3);
    }
    float dot = (a0 + a1) + (a2 + a3);
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    const float coef = on ? sB[t] * dot : 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = fmaf(-coef, w[c], x[c]);
}

// ---------------------------------------------------------------------------
// 1. 128-level adjoints -> per-half adjoints (in place for dQt / dKt)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(NT) compose_adj_kernel(const T *q, const T *k, const T *w,
                                                         const float *beta, int L, int nblk,
                                                         bool vec, float *dQt, float *dKt,
                                                         const float *dPm, const float *dSd,
                                                         float *dP64)
{
    extern __shared__ __align__(16) float sm[];
    float *sW = sm;               // [128][WLD]
    float *sBt = sW + BT * WLD;   // [128]
    float *sKa = sBt + BT;        // Ktil_a
    float *sQb = sKa + MAT;       // Qtil_b
    float *sPa = sQb + MAT;       // P_a
    float *sPb = sPa + MAT;       // P_b
    float *sDX = sPb + MAT;       // dSd[b, a]
    float *sDQb = sDX + MAT;      // dQtil[b]
    float *sDKa = sDQb + MAT;     // dKtil[a]
    float *sDP = sDKa + MAT;      // dP
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int Lp = nblk * BT;
    const long long row0 = (long long)h * L + (long long)J * BT;
    const int nvalid = min(BT, L - J * BT);
    const float *dsd = dSd + ((long long)h * nblk + J) * BT * BT;
    const long long prow = (long long)h * Lp + (long long)J * BT;
    cp_rows(sDX, dsd + (long long)HB * BT, BT);
    cp_rows(sDQb, dQt + (prow + HB) * D, D);
    cp_rows(sDKa, dKt + prow * D, D);
    cp_rows(sDP, dPm + ((long long)h * nblk + J) * D * D, D);
    {
        float4 wv[BT * D / 4 / NT];
#pragma unroll
        for (int j = 0; j < BT * D / 4 / NT; ++j) {
            const int e = tid + j * NT, r = e >> 4, c = (e & 15) * 4;
            wv[j] = r < nvalid ? ld4(w + row0 * D, D, r, c, vec) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < BT * D / 4 / NT; ++j) {
            const int e = tid + j * NT, r = e >> 4, c = (e & 15) * 4;
            *reinterpret_cast<float4 *>(sW + wx(r, c)) = wv[j];
        }
    }
    for (int r = tid; r < BT; r += NT) sBt[r] = r < nvalid ? beta[row0 + r] : 0.f;
    cp_async_wait_all();
    __syncthreads();
    // the halves' own quantities, by recurrence; lane pair (2r, 2r+1) of role g
    // holds row or column r, 32 columns each; the step index is warp-uniform
    {
        const int g = tid >> 7, r = (tid & 127) >> 1, p = tid & 1, rw = r & ~15;
        float x[32];
        if (g == 0) {  // key r of half a carried to the end of half a
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 v = r < nvalid ? ld4(k + row0 * D, D, r, 32 * p + c, vec)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                x[c] = v.x, x[c + 1] = v.y, x[c + 2] = v.z, x[c + 3] = v.w;
            }
            for (int t = rw + 1; t < HB; ++t) apply_h_half(x, sW, sBt, t, p, t > r);
#pragma unroll
            for (int c = 0; c < 32; ++c) sKa[sx(r, 32 * p + c)] = x[c];
        } else if (g == 1) {  // query 64+r of half b carried back to the start of half b
            const int i = HB + r;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 v = i < nvalid ? ld4(q + row0 * D, D, i, 32 * p + c, vec)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                x[c] = v.x, x[c + 1] = v.y, x[c + 2] = v.z, x[c + 3] = v.w;
            }
            for (int t = HB + rw + 15; t >= HB; --t) apply_h_half(x, sW, sBt, t, p, t <= i);
#pragma unroll
            for (int c = 0; c < 32; ++c) sQb[sx(r, 32 * p + c)] = x[c];
        } else {  // column r of P_a (g == 2) or P_b (g == 3)
            const int t0 = g == 2 ? 0 : HB;
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = 32 * p + c == r ? 1.f : 0.f;
            for (int t = t0; t < t0 + HB; ++t) apply_h_half(x, sW, sBt, t, p);
            float *dst = g == 2 ? sPa : sPb;
#pragma unroll
            for (int c = 0; c < 32; ++c) dst[sx(32 * p + c, r)] = x[c];
        }
    }
    __syncthreads();
    // each product goes straight from registers to global memory; every read
    // of dQt / dKt (the copies above) completed before the barrier above
    {  // dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a
        Frag f;
        mm<false, true>(f, sDQb, sPa);
        mm<false, false>(f, sDX, sKa);
        put_rows(dQt + (prow + HB) * D, D, f, nullptr, nullptr, HB);
    }
    {  // dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b
        Frag f;
        mm<false, false>(f, sDKa, sPb);
        mm<true, false>(f, sDX, sQb);
        put_rows(dKt + prow * D, D, f, nullptr, nullptr, HB);
    }
    {  // dP_a = Qtil_b^T dQtil[b] + P_b^T dP
        Frag f;
        mm<true, false>(f, sQb, sDQb);
        mm<true, false>(f, sPb, sDP);
        put_rows(dP64 + ((long long)h * 2 * nblk + 2 * J) * D * D, D, f, nullptr, nullptr, HB);
    }
    {  // dP_b = dKtil[a]^T Ktil_a + dP P_a^T
        Frag f;
        mm<true, false>(f, sDKa, sKa);
        mm<false, true>(f, sDP, sPa);
        put_rows(dP64 + ((long long)h * 2 * nblk + 2 * J + 1) * D * D, D, f, nullptr, nullptr, HB);
    }
}

// ---------------------------------------------------------------------------
// 2. UT adjoint of one 64-position half
// ---------------------------------------------------------------------------
template <typename T, typename TO>
__global__ void __launch_bounds__(NT) ut_adj64_kernel(const T *q, const T *k, const T *w,
                                                      const float *beta, int L, int nblk, bool vec,
                                                      const float *dQt, const float *dKt,
                                                      const float *dP64, const float *dSd,
                                                      TO *dq, TO *dk, TO *dw, float *dbeta)
{
    extern __shared__ __align__(16) float sm[];
    float *sW = sm, *sQ = sW + MAT, *sK = sQ + MAT, *sA = sK + MAT, *sN = sA + MAT,
          *sM = sN + MAT, *sWh = sM + MAT, *sU = sWh + MAT, *sDQ = sU + MAT, *sDK = sDQ + MAT,
          *sDP = sDK + MAT, *sDS = sDP + MAT, *sDWh = sDS + MAT, *sDU = sDWh + MAT,
          *sB = sDU + MAT;
    constexpr bool EX = std::is_same<T, bf16>::value;  // W, Q, K exact in tf32
    const int blk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int J = blk / 2, half = blk % 2;
    const int Lp = nblk * BT;
    const int pos0 = J * BT + half * HB;
    const int nvalid = min(HB, L - pos0);
    if (nvalid <= 0) return;  // a half entirely past the end: nothing to produce
    const long long row0 = (long long)h * L + pos0;
    const long long prow = (long long)h * Lp + pos0;
    cp_rows(sDQ, dQt + prow * D, D);
    cp_rows(sDK, dKt + prow * D, D);
    cp_rows(sDP, dP64 + ((long long)h * 2 * nblk + blk) * D * D, D);
    cp_rows(sDS, dSd + ((long long)h * nblk + J) * BT * BT + (long long)(half * HB) * BT + half * HB, BT);
    {
        Rows<T> rw, rq, rk;
        rw.ld(w + row0 * D, nvalid, vec);
        rq.ld(q + row0 * D, nvalid, vec);
        rk.ld(k + row0 * D, nvalid, vec);
        rw.st(sW);
        rq.st(sQ);
        rk.st(sK);
    }
    for (int r = tid; r < HB; r += NT) sB[r] = r < nvalid ? beta[row0 + r] : 0.f;
    cp_async_wait_all();
    __syncthreads();
    // forward quantities
    {
        Frag f;
        mm<false, true, EX, EX>(f, sW, sW);
        put(sA, f, 1.f, false, OUT_STRICT, sB);  // A = strictLower(D W W^T)
    }
    diag_inverse(sA);
    {
        Frag f;
        mm<false, true, EX, EX>(f, sW, sK);
        put(sN, f, 1.f, false, OUT_STRICT);  // N = strictLower(W K^T)
    }
    {
        Frag f;
        mm<false, true, EX, EX>(f, sQ, sW);
        put(sM, f, 1.f, false, OUT_LOWER);  // M = lower(Q W^T)
    }
    // [What | U] = (I + A)^{-1} D [W | N]: forward substitution, 128 right-hand sides
    for (int e = tid; e < MAT; e += NT) {
        const int r = e / HB, c = e % HB;
        sWh[sx(r, c)] = sB[r] * sW[sx(r, c)];
        sU[sx(r, c)] = sB[r] * sN[sx(r, c)];
    }
    __syncthreads();
    tri_solve<false>(sA, sWh, sU);
    // adjoint
    {
        Frag f;
        mm<true, false>(f, sM, sDQ);
        mm<false, false, EX, false>(f, sW, sDP);
        put(sDWh, f, -1.f, false, OUT_ALL);  // dWhat = -M^T dQtil - W dP
    }
    {
        Frag f;
        mm<false, true, EX, false>(f, sW, sDK);
        mm<true, false>(f, sM, sDS);
        put(sDU, f, -1.f, false, OUT_ALL);  // dU = -W dKtil^T - M^T dSd
    }
    {
        Frag f;
        mm<false, true>(f, sDQ, sWh);
        mm<false, true>(f, sDS, sU);
        put(sM, f, -1.f, false, OUT_LOWER);  // dM = lower(-dQtil What^T - dSd U^T), over M
    }
    {  // dq = dQtil + dSd K + dM W
        Frag f;
        mm<false, false, false, EX>(f, sDS, sK);
        mm<false, false, false, EX>(f, sM, sW);
        put_rows(dq + row0 * D, D, f, sDQ, nullptr, nvalid);
    }
    // dR = (I + A)^{-T} [dWhat | dU]: backward substitution (its barriers also
    // order the dq reads of sDQ before sDQ is overwritten below)
    tri_solve<true>(sA, sDWh, sDU);
    {  // dA = strictLower(-(dR_w What^T + dR_n U^T))   (into sDQ)
        Frag f;
        mm<false, true>(f, sDWh, sWh);
        mm<false, true>(f, sDU, sU);
        put(sDQ, f, -1.f, false, OUT_STRICT);
    }
    {  // G = W W^T over A (free after the solves)
        Frag f;
        mm<false, true, EX, EX>(f, sW, sW);
        put(sA, f, 1.f, false, OUT_ALL);
    }
    // dbeta_a = dR_w[a].W[a] + dR_n[a].N[a] + sum_{b<a} dA[a][b] G[a][b]; eight lanes per row
    {
        const int a = tid >> 3, part = tid & 7;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < HB / 8; ++i) {
            const int c = 8 * i + part;
            s = fmaf(sDWh[sx(a, c)], sW[sx(a, c)], s);
            s = fmaf(sDU[sx(a, c)], sN[sx(a, c)], s);
            s = fmaf(sDQ[sx(a, c)], sA[sx(a, c)], s);  // dA is zero for c >= a
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (part == 0 && a < nvalid) dbeta[row0 + a] = s;
    }
    __syncthreads();
    // dN = strictLower(D dR_n) (over dR_n); dG = strictLower(D dA) (over dA)
    scale_rows_mask(sDU, sB, OUT_STRICT);
    scale_rows_mask(sDQ, sB, OUT_STRICT);
    {  // dk = dKtil + dSd^T Q + dN^T W
        Frag f;
        mm<true, false, false, EX>(f, sDS, sQ);
        mm<true, false, false, EX>(f, sDU, sW);
        put_rows(dk + row0 * D, D, f, sDK, nullptr, nvalid);
    }
    {  // dw = D dR_w - U dKtil - What dP^T + dM^T Q + dN K + (dG + dG^T) W
        Frag f;
        mm<false, false>(f, sU, sDK, -1.f);
        mm<false, true>(f, sWh, sDP, -1.f);
        mm<true, false, false, EX>(f, sM, sQ);
        mm<false, false, false, EX>(f, sDU, sK);
        mm<false, false, false, EX>(f, sDQ, sW);
        mm<true, false, false, EX>(f, sDQ, sW);
        put_rows(dw + row0 * D, D, f, sDWh, sB, nvalid);
    }
}


template <typename T, typename TO>
cudaError_t run(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g, float *dP64,
                cudaStream_t st)
{
    const size_t smc = (BT * WLD + BT + 8 * MAT) * sizeof(float);
    const size_t smu = (14 * MAT + HB) * sizeof(float);
    auto kc = compose_adj_kernel<T>;
    auto ku = ut_adj64_kernel<T, TO>;
    cudaError_t e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smc);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ku, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smu);
    if (e != cudaSuccess) return e;
    const T *q = static_cast<const T *>(in.q), *k = static_cast<const T *>(in.k),
            *w = static_cast<const T *>(in.w);
    const bool vec = rows_vec_aligned<T>(q) && rows_vec_aligned<T>(k) && rows_vec_aligned<T>(w);
    {
        Stage s_c("ut_adj_compose", st);
        kc<<<dim3(Dm.nblk, Dm.nh), NT, smc, st>>>(q, k, w, in.beta, Dm.L, Dm.nblk, vec,
                                                  const_cast<float *>(g.dQt),
                                                  const_cast<float *>(g.dKt), g.dPm, g.dSd, dP64);
        count_launches();
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    {
        Stage s_u("ut_adj64", st);
        ku<<<dim3(2 * Dm.nblk, Dm.nh), NT, smu, st>>>(q, k, w, in.beta, Dm.L, Dm.nblk, vec, g.dQt,
                                                      g.dKt, dP64, g.dSd, static_cast<TO *>(g.dq),
                                                      static_cast<TO *>(g.dk),
                                                      static_cast<TO *>(g.dw), g.dbeta);
        count_launches();
    }
    return cudaGetLastError();
}

}  // namespace

bool prep_backward_fused_supported(const PrepDims &Dm) { return Dm.d == D; }

// dQt and dKt are overwritten (used as scratch for the per-half adjoints).
// All workspace buffers handed in (dQt, dKt, dPm, dSd, dP64) are 16-byte aligned.
cudaError_t prep_backward_fused(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g,
                                float *dP64, cudaStream_t st)
{
    if (Dm.dt == F32) return run<float, float>(Dm, in, g, dP64, st);
    if (Dm.odt == BF16) return run<bf16, bf16>(Dm, in, g, dP64, st);
    return run<bf16, float>(Dm, in, g, dP64, st);
}

}  // namespace path
