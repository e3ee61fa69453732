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

namespace path {

namespace {

constexpr int HB = 64;            // half block
constexpr int D = 64;             // head dim of this path
constexpr int NT = 512;           // 16 warps
constexpr int MAT = HB * HB;      // floats per shared 64x64 matrix
constexpr int WLD = D + 4;        // row stride of the recurrences' W (halves 4 floats apart)

enum { OUT_ALL = 0, OUT_LOWER = 1, OUT_STRICT = 2 };

// Element (r, c) of a shared 64x64 fp32 matrix. Rows are 64 floats; within a
// row the 4-column groups are permuted by XOR-ing column bits 2..4 with the
// row's low three bits, so tensor-core fragment reads hit 32 distinct banks
// whether the matrix is read row-major or transposed, and a 4-column group
// stays contiguous (16-byte copies land whole).
__device__ __forceinline__ int sx(int r, int c) { return r * HB + (c ^ (((r & 3) << 3) | (r & 4))); }

// ---------------------------------------------------------------------------
// loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Elements [c, c + 4) of row r of a row-major source with leading dimension
// ld, as floats; vec: the source rows are aligned for one vector load.
__device__ __forceinline__ float4 ld4(const float *src, long long ld, int r, int c, bool vec)
{
    const float *p = src + (long long)r * ld + c;
    if (vec) return __ldg(reinterpret_cast<const float4 *>(p));
    return make_float4(p[0], p[1], p[2], p[3]);
}

__device__ __forceinline__ float4 ld4(const bf16 *src, long long ld, int r, int c, bool vec)
{
    const bf16 *p = src + (long long)r * ld + c;
    if (vec) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
        return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
    }
    return make_float4(to_f(p[0]), to_f(p[1]), to_f(p[2]), to_f(p[3]));
}

// 64 rows of a row-major fp32 source (leading dimension ld, rows 16-byte
// aligned) into the swizzled matrix dst by asynchronous 16-byte copies.
__device__ void cp_rows(float *dst, const float *src, long long ld)
{
    for (int e = threadIdx.x; e < MAT / 4; e += NT) {
        const int r = e >> 4, c = (e & 15) * 4;
        cp_async16(dst + sx(r, c), src + (long long)r * ld + c);
    }
}

// Register-staged load of 64 rows x 64 of a row-major [*, 64] input (rows at
// or past nvalid read as zero), stored to the swizzled dst by st_rows.
template <typename T>
struct Rows {
    float4 v[MAT / 4 / NT];
    __device__ void ld(const T *src, int nvalid, bool vec)
    {
#pragma unroll
        for (int j = 0; j < MAT / 4 / NT; ++j) {
            const int e = threadIdx.x + j * NT, r = e >> 4, c = (e & 15) * 4;
            v[j] = r < nvalid ? ld4(src, D, r, c, vec) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __device__ void st(float *dst) const
    {
#pragma unroll
        for (int j = 0; j < MAT / 4 / NT; ++j) {
            const int e = threadIdx.x + j * NT, r = e >> 4, c = (e & 15) * 4;
            *reinterpret_cast<float4 *>(dst + sx(r, c)) = v[j];
        }
    }
};

// ---------------------------------------------------------------------------
// split-TF32 warp-level tensor-core products
// ---------------------------------------------------------------------------
// x = hi + lo with hi, lo TF32, and a*b ~ hi_a hi_b + hi_a lo_b + lo_a hi_b with
// fp32 accumulation, which keeps the products close to fp32 accuracy.
__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

// d += a * b, m16n8k8, tf32 inputs, fp32 accumulators
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void split_a(const float (&af)[4], uint32_t (&ah)[4], uint32_t (&al)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) split_tf32(af[i], ah[i], al[i]);
}

__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                     const float (&bf)[2])
{
    uint32_t bh[2], bl[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) split_tf32(bf[i], bh[i], bl[i]);
    mma_tf32(d, al, bh);
    mma_tf32(d, ah, bl);
    mma_tf32(d, ah, bh);
}

// Register fragment of a 64x64 product: warp w holds the 16x16 tile at rows
// 16(w>>2), columns 16(w&3), as two m16n8 accumulator tiles.
struct Frag {
    float v[2][4];
    __device__ Frag()
    {
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) v[a][b] = 0.f;
    }
};

__device__ __forceinline__ int frag_m0() { return (threadIdx.x >> 7) * 16; }
__device__ __forceinline__ int frag_n0() { return ((threadIdx.x >> 5) & 3) * 16; }

__device__ __forceinline__ unsigned smem_u32(const void *p)
{
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

// Four 8x4 fp32 blocks (each row 16 contiguous bytes at the address its lane
// gives: lanes 8j..8j+7 address rows 0..7 of block j); lane l receives element
// (l / 4, l % 4) of block j in r[j], which is the tf32 fragment layout.
__device__ __forceinline__ void ldsm_x4(float (&r)[4], unsigned addr)
{
    uint32_t u[4];
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                 : "r"(addr));
#pragma unroll
    for (int j = 0; j < 4; ++j) r[j] = __uint_as_float(u[j]);
}

// f += sgn * op(A) op(B) over the full k = 64; A, B shared (layout sx),
// op = transpose if TA / TB. EA / EB: the operand's values are exact in tf32
// (bf16 data), so its low part is zero and those products are skipped.
// Row-major fragments (A as is, B transposed) come by ldmatrix. No barrier.
template <bool TA, bool TB, bool EA = false, bool EB = false>
__device__ void mm(Frag &f, const float *A, const float *B, float sgn = 1.f)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
    const int lr = lane & 7, lm = lane >> 3;
    const int arow = m0 + lr + 8 * (lm & 1), acol = 4 * (lm >> 1);  // blocks a0..a3
    const int brow = n0 + lr + 8 * (lm >> 1), bcol = 4 * (lm & 1);  // b0, b1 of n-tile 0, then 1
    const unsigned abase = smem_u32(A), bbase = smem_u32(B);
    constexpr int UNROLL = EA || EB ? 8 : 4;  // bounded by the registers of the fully split form
#pragma unroll UNROLL
    for (int k0 = 0; k0 < HB; k0 += 8) {
        float af[4];
        if (!TA) {
            ldsm_x4(af, abase + 4u * sx(arow, k0 + acol));
        } else {
            af[0] = A[sx(k0 + tg, m0 + g)];
            af[1] = A[sx(k0 + tg, m0 + g + 8)];
            af[2] = A[sx(k0 + tg + 4, m0 + g)];
            af[3] = A[sx(k0 + tg + 4, m0 + g + 8)];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) af[i] *= sgn;
        float bq[4];
        if (TB) {
            ldsm_x4(bq, bbase + 4u * sx(brow, k0 + bcol));
        } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                bq[2 * nt] = B[sx(k0 + tg, n0 + nt * 8 + g)];
                bq[2 * nt + 1] = B[sx(k0 + tg + 4, n0 + nt * 8 + g)];
            }
        }
        uint32_t ah[4], al[4];
        if (EA) {
#pragma unroll
            for (int i = 0; i < 4; ++i) ah[i] = __float_as_uint(af[i]), al[i] = 0u;
        } else {
            split_a(af, ah, al);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if (EB)
                    bh[i] = __float_as_uint(bq[2 * nt + i]), bl[i] = 0u;
                else
                    split_tf32(bq[2 * nt + i], bh[i], bl[i]);
            }
            if (!EA) mma_tf32(f.v[nt], al, bh);
            if (!EB) mma_tf32(f.v[nt], ah, bl);
            mma_tf32(f.v[nt], ah, bh);
        }
    }
}

// C (=|+=) alpha * rs[i] * f (rs = 1 when null), masked (OUT_LOWER keeps
// j <= i, OUT_STRICT keeps j < i), then a barrier. C must not be an operand of
// the products that made f.
__device__ void put(float *C, const Frag &f, float alpha, bool accumulate, int mask,
                    const float *rs = nullptr)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = m0 + g + (q >> 1) * 8, j = n0 + nt * 8 + 2 * tg + (q & 1);
            float v = alpha * (rs ? rs[i] : 1.f) * f.v[nt][q] + (accumulate ? C[sx(i, j)] : 0.f);
            if ((mask == OUT_LOWER && j > i) || (mask == OUT_STRICT && j >= i)) v = 0.f;
            C[sx(i, j)] = v;
        }
    __syncthreads();
}

// dst[i][j] = f[i][j] + rs[i] * X[i][j] (rs = 1 when null; X may be null) for
// rows i < nvalid, dst row-major with leading dimension ld in global memory.
// No barrier.
template <typename TO>
__device__ void put_rows(TO *dst, long long ld, const Frag &f, const float *X, const float *rs,
                         int nvalid)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int i = m0 + g + hh * 8, j = n0 + nt * 8 + 2 * tg;
            if (i >= nvalid) continue;
            float v0 = f.v[nt][2 * hh], v1 = f.v[nt][2 * hh + 1];
            if (X) {
                const float r = rs ? rs[i] : 1.f;
                v0 += r * X[sx(i, j)];
                v1 += r * X[sx(i, j + 1)];
            }
            TO *p = dst + (long long)i * ld + j;
            p[0] = from_f<TO>(v0);
            p[1] = from_f<TO>(v1);
        }
}

// Overwrites each 16x16 diagonal block of the strictly lower A (whose
// diagonal blocks are otherwise unused by the solves below) with the unit
// lower triangular (I + A_cc)^{-1}, column by column by forward substitution
// (one thread per column). Ends with a barrier.
__device__ void diag_inverse(float *sA)
{
    const int tid = threadIdx.x, r0 = 16 * (tid >> 4), j = tid & 15;
    float x[16];
    if (tid < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = i == j ? 1.f : 0.f;
#pragma unroll
            for (int kk = 0; kk < i; ++kk) s = fmaf(-sA[sx(r0 + i, r0 + kk)], x[kk], s);
            x[i] = s;  // zero above the diagonal (i < j)
        }
    }
    __syncthreads();
    if (tid < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) sA[sx(r0 + i, r0 + j)] = x[i];
    }
    __syncthreads();
}

// Solves in place, per 64x128 right-hand side Z = [Z0 | Z1] (two shared
// matrices), forward (I + A) X = Z or transposed (I + A)^T X = Z, where sA
// holds the strictly lower A off the diagonal blocks and the blocks'
// inverses on them (diag_inverse). Warp w owns the 8 columns 8(w&7).. of Z0
// (w < 8) or Z1; per 16-row chunk c (in solve order) it forms
// Z_c - sum over solved chunks k of A_ck X_k, then X_c = T_c (that) with
// T_c the block inverse (transposed for the transposed system), both on the
// tensor cores.
template <bool TRANS>
__device__ void tri_solve(const float *sA, float *Z0, float *Z1)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    float *Z = warp < 8 ? Z0 : Z1;
    const int c0 = (warp & 7) * 8;
    // (i, k) entry of the system's off-diagonal blocks / of the block inverse
    auto sys = [&](int i, int k) { return TRANS ? sA[sx(k, i)] : sA[sx(i, k)]; };
    auto chunk_mma = [&](float (&acc)[4], int r0, int k0) {
        const float af[4] = {sys(r0 + g, k0 + tg), sys(r0 + g + 8, k0 + tg), sys(r0 + g, k0 + tg + 4),
                             sys(r0 + g + 8, k0 + tg + 4)};
        uint32_t ah[4], al[4];
        split_a(af, ah, al);
        const float bf[2] = {Z[sx(k0 + tg, c0 + g)], Z[sx(k0 + tg + 4, c0 + g)]};
        mma3(acc, ah, al, bf);
    };
    for (int cb = 0; cb < 4; ++cb) {
        const int r0 = TRANS ? (3 - cb) * 16 : cb * 16;
        // rows already solved: [0, r0) forward, [r0 + 16, 64) transposed
        const int s0 = TRANS ? r0 + 16 : 0, s1 = TRANS ? HB : r0;
        if (s1 > s0) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int k0 = s0; k0 < s1; k0 += 8) chunk_mma(acc, r0, k0);
#pragma unroll
            for (int q = 0; q < 4; ++q) Z[sx(r0 + g + (q >> 1) * 8, c0 + 2 * tg + (q & 1))] -= acc[q];
            __syncwarp();
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        chunk_mma(acc, r0, r0);
        chunk_mma(acc, r0, r0 + 8);
        __syncwarp();  // every lane has read the chunk before it is overwritten
#pragma unroll
        for (int q = 0; q < 4; ++q) Z[sx(r0 + g + (q >> 1) * 8, c0 + 2 * tg + (q & 1))] = acc[q];
        __syncwarp();
    }
    __syncthreads();
}

// Row-scale and mask in place: X[i][j] *= s[i] (masked entries zeroed).
__device__ void scale_rows_mask(float *X, const float *s, int mask)
{
    for (int e = threadIdx.x; e < MAT; e += NT) {
        const int i = e / HB, j = e % HB;
        float v = X[sx(i, j)] * s[i];
        if ((mask == OUT_LOWER && j > i) || (mask == OUT_STRICT && j >= i)) v = 0.f;
        X[sx(i, j)] = v;
    }
    __syncthreads();
}

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

template <typename T>
bool rows_vec_aligned(const void *p)
{
    // one vector load per 4 elements: 16 bytes (fp32) or 8 bytes (bf16); rows are 64 elements
    return (reinterpret_cast<uintptr_t>(p) % (4 * sizeof(T))) == 0;
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
