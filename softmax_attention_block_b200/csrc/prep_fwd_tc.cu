// Forward UT prep of one 128-position block on tensor cores, head dim 64.
//
// Per 64-position half h (positions s..e, H_t = I - beta_t w_t w_t^T), the UT
// transform in closed form (Paper-Notes "训练策略": T^{-1} = (I + strictLower(D W W^T))^{-1} D,
// and the full-matrix form of the diagonal-block logits):
//   A = strictLower(D W W^T), N = strictLower(W K^T), M = lower(Q W^T),
//   [What | U] = (I + A)^{-1} D [W | N]                  (one triangular solve)
//   Qtil_h = Q - M What        (queries carried back to the half's start)
//   Ktil_h = K - U^T W         (keys carried to the half's end)
//   P_h    = I - W^T What      (H_e ... H_s)
//   Sd_hh  = lower(Q K^T - M U) (logits inside the half)
// and the 128-block from its halves a (first) and b:
//   Qtil[a] = Qtil_a,  Qtil[b] = Qtil_b P_a,  Ktil[a] = Ktil_a P_b^T,  Ktil[b] = Ktil_b,
//   P = P_b P_a,  Sd = [[Sd_aa, 0], [Qtil_b Ktil_a^T, Sd_bb]].
// The same quantities as the rank-one recurrences of prep_fwd_rec.cu, as 64x64
// products in split TF32 (near fp32) and one solve per half.
#include <type_traits>

#include "prep.cuh"
#include "runtime.cuh"
#include "ut64.cuh"

namespace path {

namespace {

using namespace ut64;

// dst[i][j] = f[i][j] + X[i][j] (X may be null) + [i == j] if identity, all 64
// rows; OUT_LOWER stores zero above the diagonal. dst row-major, leading
// dimension ld, in global memory. No barrier.
template <typename TO>
__device__ void store_frag(TO *dst, long long ld, const Frag &f, const float *X, bool identity,
                           int mask)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int i = m0 + g + hh * 8, j = n0 + nt * 8 + 2 * tg;
            float v[2] = {f.v[nt][2 * hh], f.v[nt][2 * hh + 1]};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (X) v[e] += X[sx(i, j + e)];
                if (identity && i == j + e) v[e] += 1.f;
                if (mask == OUT_LOWER && j + e > i) v[e] = 0.f;
            }
            TO *p = dst + (long long)i * ld + j;
            p[0] = from_f<TO>(v[0]);
            p[1] = from_f<TO>(v[1]);
        }
}

// C = f + I (shared, layout sx), then a barrier.
__device__ void put_identity_plus(float *C, const Frag &f)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = m0 + g + (q >> 1) * 8, j = n0 + nt * 8 + 2 * tg + (q & 1);
            C[sx(i, j)] = f.v[nt][q] + (i == j ? 1.f : 0.f);
        }
    __syncthreads();
}

template <typename T, typename TM>
__global__ void __launch_bounds__(NT) prep_fwd_tc_kernel(const T *q, const T *k, const T *w,
                                                         const float *beta, int L, int nblk,
                                                         bool vec, TM *Qt, TM *Kt, TM *Pm,
                                                         float *Sd, float *halves)
{
    constexpr bool EX = std::is_same<T, bf16>::value;  // W, Q, K exact in tf32
    // bf16 inputs: single-TF32 products (the precision of the fp16 outputs of
    // this path); fp32 inputs: split TF32 (near fp32)
    constexpr bool SPLIT = !EX;
    extern __shared__ __align__(16) float sm[];
    // working set of one half, then what the composition keeps
    float *sWa = sm, *sQw = sWa + MAT, *sKw = sQw + MAT, *sA = sKw + MAT, *sM = sA + MAT,
          *sWh = sM + MAT, *sU = sWh + MAT, *sKa = sU + MAT, *sPa = sKa + MAT, *sQb = sPa + MAT,
          *sPb = sQb + MAT, *sWb = sPb + MAT, *sBa = sWb + MAT, *sBb = sBa + HB;
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int Lp = nblk * BT;
    const long long prow = (long long)h * Lp + (long long)J * BT;  // block's first row in [nh, Lp]
    float *sd = Sd + ((long long)h * nblk + J) * BT * BT;

    // both halves' inputs up front (half a keeps its keys, -> Ktil_a, in sKa and
    // half b its queries, -> Qtil_b, in sQb), so half b's loads are not exposed
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        const int pos0 = J * BT + half * HB;
        const int nvalid = max(0, min(HB, L - pos0));
        const long long row0 = (long long)h * L + pos0;
        Rows<T> rw, rq, rk;
        rw.ld(w + row0 * D, nvalid, vec);
        rq.ld(q + row0 * D, nvalid, vec);
        rk.ld(k + row0 * D, nvalid, vec);
        rw.st(half == 0 ? sWa : sWb);
        rq.st(half == 0 ? sQw : sQb);
        rk.st(half == 0 ? sKa : sKw);
        float *sB = half == 0 ? sBa : sBb;
        for (int r = tid; r < HB; r += NT) sB[r] = r < nvalid ? beta[row0 + r] : 0.f;
    }
    __syncthreads();

#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        float *sK = half == 0 ? sKa : sKw;
        float *sQ = half == 0 ? sQw : sQb;
        float *sW = half == 0 ? sWa : sWb;
        float *sB = half == 0 ? sBa : sBb;
        {
            Frag f;
            mm<false, true, EX, EX, SPLIT>(f, sW, sW);
            put(sA, f, 1.f, false, OUT_STRICT, sB);  // A = strictLower(D W W^T)
        }
        diag_inverse(sA);
        {
            Frag f;
            mm<false, true, EX, EX, SPLIT>(f, sW, sK);
            put(sU, f, 1.f, false, OUT_STRICT, sB);  // D N, N = strictLower(W K^T)
        }
        {
            Frag f;
            mm<false, true, EX, EX, SPLIT>(f, sQ, sW);
            put(sM, f, 1.f, false, OUT_LOWER);  // M = lower(Q W^T)
        }
        for (int e = tid; e < MAT; e += NT) {
            const int r = e / HB, c = e % HB;
            sWh[sx(r, c)] = sB[r] * sW[sx(r, c)];
        }
        __syncthreads();
        tri_solve<false, SPLIT>(sA, sWh, sU);  // [What | U] = (I + A)^{-1} D [W | N]
        {
            // Sd_hh = lower(Q K^T - M U); the block above the diagonal is zero
            Frag f;
            mm<false, true, EX, EX, SPLIT>(f, sQ, sK);
            mm<false, false, false, false, SPLIT>(f, sM, sU, -1.f);
            store_frag(sd + (long long)(half * HB) * BT + half * HB, BT, f, nullptr, false, OUT_LOWER);
            if (half == 0) {
                for (int e = tid; e < MAT; e += NT) sd[(long long)(e / HB) * BT + HB + e % HB] = 0.f;
            }
        }
        {
            // Qtil_h = Q - M What (in place for half b: after every read of Q above)
            Frag f;
            mm<false, false, false, false, SPLIT>(f, sM, sWh, -1.f);
            if (half == 0) {
                store_frag(Qt + prow * D, D, f, sQ, false, OUT_ALL);
            } else {
                __syncthreads();
                put(sQ, f, 1.f, true, OUT_ALL);
            }
        }
        {
            // Ktil_h = K - U^T W (in place for half a: after every read of K above)
            Frag f;
            mm<true, false, false, EX, SPLIT>(f, sU, sW, -1.f);
            if (half == 0) {
                __syncthreads();
                put(sK, f, 1.f, true, OUT_ALL);
            } else {
                store_frag(Kt + (prow + HB) * D, D, f, sK, false, OUT_ALL);
            }
        }
        {
            // P_h = I - W^T What
            Frag f;
            mm<true, false, EX, false, SPLIT>(f, sW, sWh, -1.f);
            put_identity_plus(half == 0 ? sPa : sPb, f);
        }
    }
    if (halves) {
        // Ktil_a, Qtil_b, P_a, P_b for the backward's composition adjoint
        float *dst = halves + ((long long)h * nblk + J) * 4 * MAT;
        const float *src[4] = {sKa, sQb, sPa, sPb};
#pragma unroll
        for (int m = 0; m < 4; ++m)
            for (int e = tid; e < MAT / 4; e += NT) {
                const int r = e >> 4, c = (e & 15) * 4;
                *reinterpret_cast<float4 *>(dst + m * MAT + r * HB + c) =
                    *reinterpret_cast<const float4 *>(src[m] + sx(r, c));
            }
    }
    // compose the 128-block
    {
        Frag f;
        mm<false, false, false, false, SPLIT>(f, sQb, sPa);
        store_frag(Qt + (prow + HB) * D, D, f, nullptr, false, OUT_ALL);  // Qtil_b P_a
    }
    {
        Frag f;
        mm<false, true, false, false, SPLIT>(f, sKa, sPb);
        store_frag(Kt + prow * D, D, f, nullptr, false, OUT_ALL);  // Ktil_a P_b^T
    }
    {
        Frag f;
        mm<false, false, false, false, SPLIT>(f, sPb, sPa);
        store_frag(Pm + ((long long)h * nblk + J) * D * D, D, f, nullptr, false, OUT_ALL);
    }
    {
        Frag f;
        mm<false, true, false, false, SPLIT>(f, sQb, sKa);
        store_frag(sd + (long long)HB * BT, BT, f, nullptr, false, OUT_ALL);  // Qtil_b Ktil_a^T
    }
}

template <typename T, typename TM>
cudaError_t run(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out, cudaStream_t st)
{
    const size_t smem = (12 * MAT + 2 * HB) * sizeof(float);
    auto kern = prep_fwd_tc_kernel<T, TM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const T *q = static_cast<const T *>(in.q), *k = static_cast<const T *>(in.k),
            *w = static_cast<const T *>(in.w);
    const bool vec = rows_vec_aligned<T>(q) && rows_vec_aligned<T>(k) && rows_vec_aligned<T>(w);
    kern<<<dim3(Dm.nblk, Dm.nh), NT, smem, st>>>(q, k, w, in.beta, Dm.L, Dm.nblk, vec,
                                                 static_cast<TM *>(out.Qt), static_cast<TM *>(out.Kt),
                                                 static_cast<TM *>(out.Pm), out.Sd, out.halves);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool prep_forward_tc_supported(const PrepDims &Dm) { return Dm.d == D; }

cudaError_t prep_forward_tc(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out,
                            cudaStream_t st)
{
    if (Dm.dt == F32) return run<float, float>(Dm, in, out, st);
    return run<bf16, f16>(Dm, in, out, st);
}

}  // namespace path
