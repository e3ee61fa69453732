// The decode cache a prefill leaves. After positions 0..L-1 the in-place
// updated key cache holds, in row j, H_{L-1} ... H_{j+1} k_j (Paper-Notes
// "训练策略", inference paragraph). The forward already formed, for every key
// block J, the keys carried through all blocks before the last one,
//   Khat_{last,J} = Ktil_J P_{J+1}^T ... P_{last-1}^T,
// so one more block product finishes the transport:
//   cache_J    = Khat_{last,J} P_last^T   (J < last),
//   cache_last = Ktil_last                 (already carried to position L-1:
//                                           H is the identity past L),
// i.e. the right-to-left scan of gist.science section 3 taken one block
// further on the key side. Values are copied as they are; with the forget gate
// each row also gets its logit bias g_j = c_{L-1} - c_j (Paper-Notes "PaTH-FoX
// 扩展"), which a gated decode step then carries forward in place.
//
// One CTA per (key block, head): X (128 x d) and P_last^T in shared memory as
// fp32, each thread one row and half of the columns, fp32 accumulation.
#include "attn.cuh"
#include "runtime.cuh"

namespace path {

namespace {

constexpr int CT = 256;

template <typename T>
struct Elems16 {
    static constexpr int N = 16 / sizeof(T);
};

template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &u, float *f)
{
    if constexpr (sizeof(T) == 4) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    } else {
        const T *h = reinterpret_cast<const T *>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = to_f(h[i]);
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack16(const float *f)
{
    uint4 u;
    T *h = reinterpret_cast<T *>(&u);
#pragma unroll
    for (int i = 0; i < Elems16<T>::N; ++i) h[i] = from_f<T>(f[i]);
    return u;
}

template <int D>
struct CacheSmem {
    static constexpr int XS = D + 1;  // row stride of X: rows on distinct banks
    static constexpr int FLOATS = D * D + BT * XS;
};

// TM: type of the forward's transported keys and block products; TC: type of
// the caches (the call's input type).
template <typename TM, typename TC, int D>
__global__ void __launch_bounds__(CT) prefill_cache_kernel(CacheArgs a)
{
    using S = CacheSmem<D>;
    constexpr int VM = Elems16<TM>::N, VC = Elems16<TC>::N;
    extern __shared__ __align__(16) float csm[];
    float *sPt = csm;          // sPt[e * D + c] = P_last[c][e]
    float *sX = csm + D * D;   // sX[r * XS + e]
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int last = a.nblk - 1, Lp = a.nblk * BT;
    const int row0 = J * BT;
    const int nvalid = min(BT, a.L - row0);
    const bool transport = J < last;
    const long long npairs = (long long)a.nblk * (a.nblk - 1) / 2;
    const TM *X = transport
                      ? static_cast<const TM *>(a.Khat) +
                            (h * npairs + (long long)last * (last - 1) / 2 + J) * BT * D
                      : static_cast<const TM *>(a.Kt) + ((long long)h * Lp + row0) * D;

    for (int i = tid; i < BT * D / VM; i += CT) {
        float f[VM];
        unpack16<TM>(reinterpret_cast<const uint4 *>(X)[i], f);
        const int r = i * VM / D, e0 = i * VM % D;
#pragma unroll
        for (int k = 0; k < VM; ++k) sX[r * S::XS + e0 + k] = f[k];
    }
    if (transport) {
        const TM *P = static_cast<const TM *>(a.Pm) + ((long long)h * a.nblk + last) * D * D;
        for (int i = tid; i < D * D / VM; i += CT) {
            float f[VM];
            unpack16<TM>(reinterpret_cast<const uint4 *>(P)[i], f);
            const int c = i * VM / D, e0 = i * VM % D;
#pragma unroll
            for (int k = 0; k < VM; ++k) sPt[(e0 + k) * D + c] = f[k];
        }
    }
    // values and gate biases of the block's valid rows
    {
        const long long src = ((long long)h * a.L + row0) * D / VC;
        const long long dst = ((long long)h * a.capacity + row0) * D / VC;
        const uint4 *vs = reinterpret_cast<const uint4 *>(a.v);
        uint4 *vd = reinterpret_cast<uint4 *>(a.v_cache);
        for (int i = tid; i < nvalid * D / VC; i += CT) vd[dst + i] = vs[src + i];
        if (a.g_cache) {
            const float *c = a.c + (long long)h * Lp;
            const float cL = c[a.L - 1];
            for (int r = tid; r < nvalid; r += CT)
                a.g_cache[(long long)h * a.capacity + row0 + r] = cL - c[row0 + r];
        }
    }
    __syncthreads();

    // thread: row r, columns [c0, c0 + D/2); a warp shares c0, so the P reads
    // are broadcasts and the X reads hit 32 distinct banks
    constexpr int NC = D / 2;
    const int r = tid % BT, c0 = (tid / BT) * NC;
    float acc[NC];
    if (transport) {
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = 0.f;
#pragma unroll 4
        for (int e = 0; e < D; ++e) {
            const float x = sX[r * S::XS + e];
            const float4 *p = reinterpret_cast<const float4 *>(sPt + e * D + c0);
#pragma unroll
            for (int c4 = 0; c4 < NC / 4; ++c4) {
                const float4 pv = p[c4];
                acc[4 * c4 + 0] = fmaf(x, pv.x, acc[4 * c4 + 0]);
                acc[4 * c4 + 1] = fmaf(x, pv.y, acc[4 * c4 + 1]);
                acc[4 * c4 + 2] = fmaf(x, pv.z, acc[4 * c4 + 2]);
                acc[4 * c4 + 3] = fmaf(x, pv.w, acc[4 * c4 + 3]);
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = sX[r * S::XS + c0 + c];
    }
    if (r < nvalid) {
        uint4 *kd = reinterpret_cast<uint4 *>(static_cast<TC *>(a.k_cache) +
                                              ((long long)h * a.capacity + row0 + r) * D + c0);
#pragma unroll
        for (int c = 0; c < NC / VC; ++c) kd[c] = pack16<TC>(acc + c * VC);
    }
}

template <typename TM, typename TC, int D>
cudaError_t run(const CacheArgs &a, cudaStream_t st)
{
    const size_t smem = CacheSmem<D>::FLOATS * sizeof(float);
    auto k = prefill_cache_kernel<TM, TC, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nblk, a.nh), CT, smem, st>>>(a);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

cudaError_t prefill_cache(const CacheArgs &a, Types t, int d, cudaStream_t st)
{
    if (t.in == F32) {
        if (d == 64) return run<float, float, 64>(a, st);
        if (d == 128) return run<float, float, 128>(a, st);
    } else {
        if (d == 64) return run<f16, bf16, 64>(a, st);
        if (d == 128) return run<f16, bf16, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace path
