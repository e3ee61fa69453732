// Building blocks of the 64-position UT kernels (head dim 64): shared fp32
// 64x64 matrices in an XOR-swizzled layout, asynchronous and vector loads,
// products on the warp-level tensor cores in split TF32, and triangular
// solves with precomputed 16x16 diagonal-block inverses. All of it assumes a
// CTA of NT = 512 threads (16 warps).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace path {
namespace ut64 {
namespace {

constexpr int HB = 64;            // half block
constexpr int D = 64;             // head dim of this path
constexpr int NT = 512;           // 16 warps
constexpr int MAT = HB * HB;      // floats per shared 64x64 matrix

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
    // nearest TF32 value (ties away from zero) by integer arithmetic on the
    // ALU pipe: add half of the 13 dropped mantissa bits' range, then clear them
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
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
// op = transpose if TA / TB. SPLIT: split TF32 (near fp32); otherwise every
// operand is rounded to TF32 once (one product per pair, fp16-class
// accuracy). EA / EB: the operand's values are exact in tf32 (bf16 data), so
// its low part is zero and those products are skipped. Row-major fragments
// (A as is, B transposed) come by ldmatrix. No barrier.
template <bool TA, bool TB, bool EA = false, bool EB = false, bool SPLIT = true>
__device__ void mm(Frag &f, const float *A, const float *B, float sgn = 1.f)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, tg = lane & 3;
    const int m0 = frag_m0(), n0 = frag_n0();
    const int lr = lane & 7, lm = lane >> 3;
    const int arow = m0 + lr + 8 * (lm & 1), acol = 4 * (lm >> 1);  // blocks a0..a3
    const int brow = n0 + lr + 8 * (lm >> 1), bcol = 4 * (lm & 1);  // b0, b1 of n-tile 0, then 1
    const unsigned abase = smem_u32(A), bbase = smem_u32(B);
    constexpr int UNROLL = EA || EB || !SPLIT ? 8 : 4;  // bounded by the registers of the split form
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
        } else if (SPLIT) {
            split_a(af, ah, al);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) ah[i] = to_tf32(af[i]), al[i] = 0u;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if (EB)
                    bh[i] = __float_as_uint(bq[2 * nt + i]), bl[i] = 0u;
                else if (SPLIT)
                    split_tf32(bq[2 * nt + i], bh[i], bl[i]);
                else
                    bh[i] = to_tf32(bq[2 * nt + i]), bl[i] = 0u;
            }
            if (SPLIT && !EA) mma_tf32(f.v[nt], al, bh);
            if (SPLIT && !EB) mma_tf32(f.v[nt], ah, bl);
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
template <bool TRANS, bool SPLIT = true>
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
        const float bf[2] = {Z[sx(k0 + tg, c0 + g)], Z[sx(k0 + tg + 4, c0 + g)]};
        if (SPLIT) {
            uint32_t ah[4], al[4];
            split_a(af, ah, al);
            mma3(acc, ah, al, bf);
        } else {
            const uint32_t ah[4] = {to_tf32(af[0]), to_tf32(af[1]), to_tf32(af[2]), to_tf32(af[3])};
            const uint32_t bh[2] = {to_tf32(bf[0]), to_tf32(bf[1])};
            mma_tf32(acc, ah, bh);
        }
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


template <typename T>
inline bool rows_vec_aligned(const void *p)
{
    // one vector load per 4 elements: 16 bytes (fp32) or 8 bytes (bf16); rows are 64 elements
    return (reinterpret_cast<uintptr_t>(p) % (4 * sizeof(T))) == 0;
}

}  // namespace
}  // namespace ut64
}  // namespace path
