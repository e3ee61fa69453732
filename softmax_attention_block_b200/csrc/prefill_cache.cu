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
// One CTA per (key block, head). With fp16 tiles (the bf16 paths) the product
// runs on the tensor cores: mma.sync m16n8k16 with fp16 operands and fp32
// accumulation (the products of fp16 values are exact in fp32, as in the
// chain that made the tiles), one warp per 16 rows, the results staged in the
// warp's own rows of shared memory and stored as 16-byte rows. With fp32 tiles
// it runs in fp32 on the CUDA cores (each thread one row, half the columns).
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

// values and gate biases of one block's valid rows (both kernels)
template <typename TC, int D>
__device__ void copy_values_and_bias(const CacheArgs &a, int h, int row0, int nvalid)
{
    constexpr int VC = Elems16<TC>::N;
    const long long src = ((long long)h * a.L + row0) * D / VC;
    const long long dst = ((long long)h * a.capacity + row0) * D / VC;
    const uint4 *vs = reinterpret_cast<const uint4 *>(a.v);
    uint4 *vd = reinterpret_cast<uint4 *>(a.v_cache);
    for (int i = threadIdx.x; i < nvalid * D / VC; i += CT) vd[dst + i] = vs[src + i];
    if (a.g_cache) {
        const float *c = a.c + (long long)h * a.nblk * BT;
        const float cL = c[a.L - 1];
        for (int r = threadIdx.x; r < nvalid; r += CT)
            a.g_cache[(long long)h * a.capacity + row0 + r] = cL - c[row0 + r];
    }
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
    constexpr int VM = Elems16<TM>::N, VC = Elems16<TC>::N;  // elements per 16 bytes
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
    copy_values_and_bias<TC, D>(a, h, row0, nvalid);
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

__device__ __forceinline__ void mma_f16_16816(float *c, const uint32_t *a, const uint32_t *b)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int D>
struct MmaSmem {
    static constexpr int S = D + 8;  // row stride in halves: 16-byte rows, fragment loads
                                     // of 8 rows x 4 words fall on 32 distinct banks
    static constexpr int HALVES = (BT + D) * S;
};

// fp16 tiles -> bf16 cache, on the tensor cores
template <int D>
__global__ void __launch_bounds__(CT) prefill_cache_mma_kernel(CacheArgs a)
{
    using S = MmaSmem<D>;
    extern __shared__ __align__(16) f16 hsm[];
    f16 *sX = hsm;              // [BT][S]: the tile, then the warp's output rows (bf16)
    f16 *sP = hsm + BT * S::S;  // [D][S]: P_last as stored, row c = P[c][:]
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tg = lane & 3;
    const int last = a.nblk - 1, Lp = a.nblk * BT;
    const int row0 = J * BT;
    const int nvalid = min(BT, a.L - row0);
    const bool transport = J < last;
    const long long npairs = (long long)a.nblk * (a.nblk - 1) / 2;
    const f16 *X = transport
                       ? static_cast<const f16 *>(a.Khat) +
                             (h * npairs + (long long)last * (last - 1) / 2 + J) * BT * D
                       : static_cast<const f16 *>(a.Kt) + ((long long)h * Lp + row0) * D;
    constexpr int RV = D / 8;  // 16-byte vectors per row
    for (int i = tid; i < BT * RV; i += CT)
        *reinterpret_cast<uint4 *>(sX + (i / RV) * S::S + (i % RV) * 8) =
            reinterpret_cast<const uint4 *>(X)[i];
    if (transport) {
        const f16 *P = static_cast<const f16 *>(a.Pm) + ((long long)h * a.nblk + last) * D * D;
        for (int i = tid; i < D * RV; i += CT)
            *reinterpret_cast<uint4 *>(sP + (i / RV) * S::S + (i % RV) * 8) =
                reinterpret_cast<const uint4 *>(P)[i];
    }
    copy_values_and_bias<bf16, D>(a, h, row0, nvalid);
    __syncthreads();

    // warp w: rows [16w, 16w + 16), all D columns; out = X P^T, i.e. B[k][n] = P[n][k]
    const int m0 = warp * 16;
    uint32_t *xw = reinterpret_cast<uint32_t *>(sX);
    const uint32_t *pw = reinterpret_cast<const uint32_t *>(sP);
    constexpr int SW = S::S / 2;  // row stride in 32-bit words
    if (transport) {
        float acc[D / 8][4];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int kw = ks * 8 + tg;  // word of columns (16 ks + 2 tg, +1)
            uint32_t af[4] = {xw[(m0 + g) * SW + kw], xw[(m0 + g + 8) * SW + kw],
                              xw[(m0 + g) * SW + kw + 4], xw[(m0 + g + 8) * SW + kw + 4]};
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                const uint32_t bf[2] = {pw[(nt * 8 + g) * SW + kw], pw[(nt * 8 + g) * SW + kw + 4]};
                mma_f16_16816(acc[nt], af, bf);
            }
        }
        __syncwarp();  // every lane's reads of the warp's rows are done
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[nt][0], acc[nt][1]);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[nt][2], acc[nt][3]);
            xw[(m0 + g) * SW + nt * 4 + tg] = *reinterpret_cast<const uint32_t *>(&lo);
            xw[(m0 + g + 8) * SW + nt * 4 + tg] = *reinterpret_cast<const uint32_t *>(&hi);
        }
    } else {
        // the last block's keys are already carried to position L-1: fp16 -> bf16
        for (int i = lane; i < 16 * D / 2; i += 32) {
            const int r = m0 + i / (D / 2), w2 = i % (D / 2);
            const __half2 v = *reinterpret_cast<const __half2 *>(&xw[r * SW + w2]);
            const __nv_bfloat162 b = __float22bfloat162_rn(__half22float2(v));
            xw[r * SW + w2] = *reinterpret_cast<const uint32_t *>(&b);
        }
    }
    __syncwarp();
    bf16 *kc = static_cast<bf16 *>(a.k_cache) + ((long long)h * a.capacity + row0) * D;
    for (int i = lane; i < 16 * RV; i += 32) {
        const int r = m0 + i / RV;
        if (r < nvalid)
            reinterpret_cast<uint4 *>(kc + (long long)r * D)[i % RV] =
                *reinterpret_cast<const uint4 *>(sX + r * S::S + (i % RV) * 8);
    }
}

template <int D>
cudaError_t run_mma(const CacheArgs &a, cudaStream_t st)
{
    const size_t smem = MmaSmem<D>::HALVES * sizeof(f16);
    auto k = prefill_cache_mma_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nblk, a.nh), CT, smem, st>>>(a);
    count_launches();
    return cudaGetLastError();
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
        if (d == 64) return run_mma<64>(a, st);
        if (d == 128) return run_mma<128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace path
