// Batched small GEMM over the (head, block) grid: the building block of the
// per-block UT transform and its adjoint. fp32 SIMT arithmetic: these
// products involve T^{-1} and its adjoints, which stay in fp32.
#include "common.cuh"
#include "runtime.cuh"

namespace path {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__device__ __forceinline__ float op_elem(const Operand &o, long long base, int r, int c, int blk,
                                         int rows, int cols)
{
    if (r >= rows || c >= cols || o.p == nullptr) return 0.f;
    const int sr = o.trans ? c : r;
    const int sc = o.trans ? r : c;
    if (o.mask == MASK_LOWER && sc > sr) return 0.f;
    if (o.mask == MASK_STRICT_LOWER && sc >= sr) return 0.f;
    if (o.seq >= 0 && blk * BT + sr >= o.seq) return 0.f;
    return load_as_f(o.p, o.dt, base + (long long)sr * o.ld + sc);
}

__global__ void __launch_bounds__(256, 4) gemm_batched_kernel(GemmArgs g)
{
    __shared__ float As[TK][TM + 1];
    __shared__ float Bs[TK][TN + 1];
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    for (int z = blockIdx.z; z < g.batch; z += gridDim.z) {
    const int h = z / g.nblk, blk = z % g.nblk;
    float acc[4][4] = {};

    for (int t = 0; t < g.nterms; ++t) {
        const Term &T = g.t[t];
        const long long abase = (long long)h * T.a.sh + (long long)blk * T.a.sb;
        const long long bbase = (long long)h * T.b.sh + (long long)blk * T.b.sb;
        float part[4][4] = {};
        for (int k0 = 0; k0 < g.K; k0 += TK) {
            // consecutive threads take consecutive stored elements (coalesced)
            if (T.a.trans) {  // stored [k][m]
#pragma unroll 1
                for (int e = threadIdx.x; e < TK * TM; e += 256) {
                    const int kk = e / TM, mm = e % TM;
                    As[kk][mm] = op_elem(T.a, abase, m0 + mm, k0 + kk, blk, g.M, g.K);
                }
            } else {          // stored [m][k]
#pragma unroll 1
                for (int e = threadIdx.x; e < TK * TM; e += 256) {
                    const int kk = e % TK, mm = e / TK;
                    As[kk][mm] = op_elem(T.a, abase, m0 + mm, k0 + kk, blk, g.M, g.K);
                }
            }
            if (T.b.trans) {  // stored [n][k]
#pragma unroll 1
                for (int e = threadIdx.x; e < TK * TN; e += 256) {
                    const int kk = e % TK, nn = e / TK;
                    Bs[kk][nn] = op_elem(T.b, bbase, k0 + kk, n0 + nn, blk, g.K, g.N);
                }
            } else {          // stored [k][n]
#pragma unroll 1
                for (int e = threadIdx.x; e < TK * TN; e += 256) {
                    const int kk = e / TN, nn = e % TN;
                    Bs[kk][nn] = op_elem(T.b, bbase, k0 + kk, n0 + nn, blk, g.K, g.N);
                }
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < TK; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) part[i][j] = fmaf(a[i], b[j], part[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(T.alpha, part[i][j], acc[i][j]);
    }

    const long long cbase = (long long)h * g.csh + (long long)blk * g.csb;
    const long long ebase = (long long)h * g.addend.sh + (long long)blk * g.addend.sb;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + ty * 4 + i;
        if (r >= g.M) continue;
        if (g.c_seq >= 0 && blk * BT + r >= g.c_seq) continue;
        float rs = 1.f;
        if (g.rowscale) {
            rs = (g.rs_seq >= 0 && blk * BT + r >= g.rs_seq)
                     ? 0.f
                     : g.rowscale[(long long)h * g.rs_sh + (long long)blk * g.rs_sb + r];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = n0 + tx * 4 + j;
            if (c >= g.N) continue;
            float v = acc[i][j] * rs;
            if (g.addend.p) v += g.gamma * op_elem(g.addend, ebase, r, c, blk, g.M, g.N);
            if (g.add_identity && r == c) v += 1.f;
            if ((g.outmask == MASK_LOWER && c > r) || (g.outmask == MASK_STRICT_LOWER && c >= r))
                v = 0.f;
            store_from_f(g.c, g.cdt, cbase + (long long)r * g.ldc + c, v);
        }
    }
    }  // batch loop
}

}  // namespace

cudaError_t gemm_batched(const GemmArgs &g, cudaStream_t stream)
{
    dim3 grid(ceil_div(g.N, TN), ceil_div(g.M, TM), g.batch < 65535 ? g.batch : 65535);
    gemm_batched_kernel<<<grid, 256, 0, stream>>>(g);
    count_launches();
    return cudaGetLastError();
}

}  // namespace path
