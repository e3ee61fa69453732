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
//    The halves' quantities are the ones the forward's UT prep computed and
//    left in the workspace.
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

// ---------------------------------------------------------------------------
// 1. 128-level adjoints -> per-half adjoints (in place for dQt / dKt)
// ---------------------------------------------------------------------------
// SPLIT: split-TF32 products (fp32 inputs); otherwise single TF32 (bf16 inputs).
template <bool SPLIT>
__global__ void __launch_bounds__(NT) compose_adj_kernel(const float *halves, int nblk, float *dQt,
                                                         float *dKt, const float *dPm,
                                                         const float *dSd, float *dP64)
{
    extern __shared__ __align__(16) float sm[];
    float *sKa = sm;              // Ktil_a
    float *sQb = sKa + MAT;       // Qtil_b
    float *sPa = sQb + MAT;       // P_a
    float *sPb = sPa + MAT;       // P_b
    float *sDX = sPb + MAT;       // dSd[b, a]
    float *sDQb = sDX + MAT;      // dQtil[b]
    float *sDKa = sDQb + MAT;     // dKtil[a]
    float *sDP = sDKa + MAT;      // dP
    const int J = blockIdx.x, h = blockIdx.y;
    const int Lp = nblk * BT;
    const float *hv = halves + ((long long)h * nblk + J) * 4 * MAT;
    const float *dsd = dSd + ((long long)h * nblk + J) * BT * BT;
    const long long prow = (long long)h * Lp + (long long)J * BT;
    // the halves' own quantities, as the forward's UT prep left them
    cp_rows(sKa, hv, HB);
    cp_rows(sQb, hv + MAT, HB);
    cp_rows(sPa, hv + 2 * MAT, HB);
    cp_rows(sPb, hv + 3 * MAT, HB);
    cp_rows(sDX, dsd + (long long)HB * BT, BT);
    cp_rows(sDQb, dQt + (prow + HB) * D, D);
    cp_rows(sDKa, dKt + prow * D, D);
    cp_rows(sDP, dPm + ((long long)h * nblk + J) * D * D, D);
    cp_async_wait_all();
    __syncthreads();
    // each product goes straight from registers to global memory; every read
    // of dQt / dKt (the copies above) completed before the barrier above
    {  // dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a
        Frag f;
        mm<false, true, false, false, SPLIT>(f, sDQb, sPa);
        mm<false, false, false, false, SPLIT>(f, sDX, sKa);
        put_rows(dQt + (prow + HB) * D, D, f, nullptr, nullptr, HB);
    }
    {  // dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b
        Frag f;
        mm<false, false, false, false, SPLIT>(f, sDKa, sPb);
        mm<true, false, false, false, SPLIT>(f, sDX, sQb);
        put_rows(dKt + prow * D, D, f, nullptr, nullptr, HB);
    }
    {  // dP_a = Qtil_b^T dQtil[b] + P_b^T dP
        Frag f;
        mm<true, false, false, false, SPLIT>(f, sQb, sDQb);
        mm<true, false, false, false, SPLIT>(f, sPb, sDP);
        put_rows(dP64 + ((long long)h * 2 * nblk + 2 * J) * D * D, D, f, nullptr, nullptr, HB);
    }
    {  // dP_b = dKtil[a]^T Ktil_a + dP P_a^T
        Frag f;
        mm<true, false, false, false, SPLIT>(f, sDKa, sKa);
        mm<false, true, false, false, SPLIT>(f, sDP, sPa);
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
    // bf16 inputs: single-TF32 products (the precision of the fp16
    // intermediates of this path); fp32 inputs: split TF32 (near fp32)
    constexpr bool SPLIT = !EX;
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
        mm<false, true, EX, EX, SPLIT>(f, sW, sW);
        put(sA, f, 1.f, false, OUT_STRICT, sB);  // A = strictLower(D W W^T)
    }
    diag_inverse(sA);
    {
        Frag f;
        mm<false, true, EX, EX, SPLIT>(f, sW, sK);
        put(sN, f, 1.f, false, OUT_STRICT);  // N = strictLower(W K^T)
    }
    {
        Frag f;
        mm<false, true, EX, EX, SPLIT>(f, sQ, sW);
        put(sM, f, 1.f, false, OUT_LOWER);  // M = lower(Q W^T)
    }
    // [What | U] = (I + A)^{-1} D [W | N]: forward substitution, 128 right-hand sides
    for (int e = tid; e < MAT; e += NT) {
        const int r = e / HB, c = e % HB;
        sWh[sx(r, c)] = sB[r] * sW[sx(r, c)];
        sU[sx(r, c)] = sB[r] * sN[sx(r, c)];
    }
    __syncthreads();
    tri_solve<false, SPLIT>(sA, sWh, sU);
    // adjoint
    {
        Frag f;
        mm<true, false, false, false, SPLIT>(f, sM, sDQ);
        mm<false, false, EX, false, SPLIT>(f, sW, sDP);
        put(sDWh, f, -1.f, false, OUT_ALL);  // dWhat = -M^T dQtil - W dP
    }
    {
        Frag f;
        mm<false, true, EX, false, SPLIT>(f, sW, sDK);
        mm<true, false, false, false, SPLIT>(f, sM, sDS);
        put(sDU, f, -1.f, false, OUT_ALL);  // dU = -W dKtil^T - M^T dSd
    }
    {
        Frag f;
        mm<false, true, false, false, SPLIT>(f, sDQ, sWh);
        mm<false, true, false, false, SPLIT>(f, sDS, sU);
        put(sM, f, -1.f, false, OUT_LOWER);  // dM = lower(-dQtil What^T - dSd U^T), over M
    }
    {  // dq = dQtil + dSd K + dM W
        Frag f;
        mm<false, false, false, EX, SPLIT>(f, sDS, sK);
        mm<false, false, false, EX, SPLIT>(f, sM, sW);
        put_rows(dq + row0 * D, D, f, sDQ, nullptr, nvalid);
    }
    // dR = (I + A)^{-T} [dWhat | dU]: backward substitution (its barriers also
    // order the dq reads of sDQ before sDQ is overwritten below)
    tri_solve<true, SPLIT>(sA, sDWh, sDU);
    {  // dA = strictLower(-(dR_w What^T + dR_n U^T))   (into sDQ)
        Frag f;
        mm<false, true, false, false, SPLIT>(f, sDWh, sWh);
        mm<false, true, false, false, SPLIT>(f, sDU, sU);
        put(sDQ, f, -1.f, false, OUT_STRICT);
    }
    {  // G = W W^T over A (free after the solves)
        Frag f;
        mm<false, true, EX, EX, SPLIT>(f, sW, sW);
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
        mm<true, false, false, EX, SPLIT>(f, sDS, sQ);
        mm<true, false, false, EX, SPLIT>(f, sDU, sW);
        put_rows(dk + row0 * D, D, f, sDK, nullptr, nvalid);
    }
    {  // dw = D dR_w - U dKtil - What dP^T + dM^T Q + dN K + (dG + dG^T) W
        Frag f;
        mm<false, false, false, false, SPLIT>(f, sU, sDK, -1.f);
        mm<false, true, false, false, SPLIT>(f, sWh, sDP, -1.f);
        mm<true, false, false, EX, SPLIT>(f, sM, sQ);
        mm<false, false, false, EX, SPLIT>(f, sDU, sK);
        mm<false, false, false, EX, SPLIT>(f, sDQ, sW);
        mm<true, false, false, EX, SPLIT>(f, sDQ, sW);
        put_rows(dw + row0 * D, D, f, sDWh, sB, nvalid);
    }
}


template <typename T, typename TO>
cudaError_t run(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g, float *dP64,
                cudaStream_t st)
{
    const size_t smc = 8 * MAT * sizeof(float);
    const size_t smu = (14 * MAT + HB) * sizeof(float);
    auto kc = compose_adj_kernel<std::is_same<T, float>::value>;
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
        kc<<<dim3(Dm.nblk, Dm.nh), NT, smc, st>>>(g.halves, Dm.nblk, const_cast<float *>(g.dQt),
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
