// tcgen05 building blocks of the per-block UT kernels (head dim 64).
//
// A 128-position block is two 64-position halves a and b. Every per-half
// product is a 64 x 64 x 64 tensor-core MMA (M = 64) whose accumulator sits in
// tensor memory at lane offset 0 (half a) or 16 (half b) of each 32-lane
// quarter, sharing columns: rows 16q..16q+15 of half a are lanes 32q..32q+15,
// those of half b lanes 32q+16..32q+31. A warp reading its quarter with the
// 32x32b shape therefore gets one row of half a (threads 0-15) and one row of
// half b (threads 16-31).
//
// Operands are 64 x 64 fp16 tiles in shared memory, 128-byte swizzled
// (tc::sw128_offset), 8 KB each, stored row-major; a product may read either
// operand as stored or transposed (descriptor major-ness), so no transposed
// copies are made.
#pragma once
#include "tc.cuh"

namespace path {
namespace uttc {

constexpr int HB = 64;            // positions per half block
constexpr uint32_t TILE = 8192;   // bytes of one 64 x 64 16-bit tile

// A operand: as stored (rows are M, K-major) or transposed (rows are K, MN-major)
enum OpA { A_N = 0, A_T = 1 };
// B operand: D = A . stored^T (rows are N, K-major) or D = A . stored (rows are K, MN-major)
enum OpB { B_T = 0, B_N = 1 };

// One thread: D[64 x 64 nt] (+)= opA(A) opB(B) over K = 64, fp16 operands,
// fp32 accumulation (ab: both operands fp16, or both bf16). d: tensor-memory address (lane offset selects the half);
// a, b: shared addresses of the tiles; the nt column groups of B are tiles at
// stride bstride (B_T needs bstride == TILE: consecutive rows).
__device__ __forceinline__ void mma64(uint32_t d, uint32_t a, int opa, uint32_t b, int opb, int nt,
                                      uint32_t bstride, bool accumulate, int ab = tc::AB_F16)
{
    const uint32_t id = tc::idesc_f16(64, 64 * nt, ab, opa, opb);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = opa == A_N ? tc::desc_sw128(a + kk * 32, 16, 1024)
                                       : tc::desc_sw128(a + kk * 2048, TILE, 1024);
        const uint64_t bd = opb == B_T ? tc::desc_sw128(b + kk * 32, 16, 1024)
                                       : tc::desc_sw128(b + kk * 2048, bstride, 1024);
        tc::mma_ss(d, ad, bd, id, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// Tensor-memory address of column `col` for half h (0: a, 1: b) as an MMA
// destination.
__device__ __forceinline__ uint32_t dst(uint32_t tbase, int h, int col)
{
    return tbase + ((uint32_t)(16 * h) << 16) + (uint32_t)col;
}

// The calling thread's place in the epilogues (CTA of 256 threads): warp w
// reads lane quarter w % 4 and the 32-column half w / 4 of each 64-column
// group; thread t of the warp holds row 16 (w % 4) + t % 16 of half t / 16.
struct Me {
    int h, r, cg;
    uint32_t lane_off;
    __device__ Me()
    {
        const int w = threadIdx.x >> 5, t = threadIdx.x & 31;
        h = t >> 4;
        r = 16 * (w & 3) + (t & 15);
        cg = w >> 2;
        lane_off = (uint32_t)(32 * (w & 3)) << 16;
    }
    // 32 fp32 values of this thread's row: columns [col + 32 cg, col + 32 cg + 32)
    __device__ __forceinline__ void ld(uint32_t tbase, int col, float (&v)[32]) const
    {
        tc::tmem_ld32(tbase + lane_off + (uint32_t)(col + 32 * cg), v);
    }
};

// Row r, columns [c0, c0 + 32) of a tile, from 32 fp32 values (rounded to fp16).
__device__ __forceinline__ void st_tile_f16(uint8_t *tile, int r, int c0, const float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 u;
        __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) hh[i] = __floats2half2_rn(v[8 * j + 2 * i], v[8 * j + 2 * i + 1]);
        *reinterpret_cast<uint4 *>(tile + tc::sw128_offset(r, c0 + 8 * j)) = u;
    }
}

// Row r, columns [c0, c0 + 32) of a bf16 tile as floats.
__device__ __forceinline__ void ld_tile_bf16(const uint8_t *tile, int r, int c0, float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + tc::sw128_offset(r, c0 + 8 * j));
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(b[i]);
            v[8 * j + 2 * i] = f.x;
            v[8 * j + 2 * i + 1] = f.y;
        }
    }
}

// Row r, columns [c0, c0 + 32) of an fp16 tile as floats.
__device__ __forceinline__ void ld_tile_f16(const uint8_t *tile, int r, int c0, float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + tc::sw128_offset(r, c0 + 8 * j));
        const __half2 *b = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(b[i]);
            v[8 * j + 2 * i] = f.x;
            v[8 * j + 2 * i + 1] = f.y;
        }
    }
}

// 32 values to global memory (16-byte aligned destination).
__device__ __forceinline__ void st_global(f16 *dst, const float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 u;
        __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) hh[i] = __floats2half2_rn(v[8 * j + 2 * i], v[8 * j + 2 * i + 1]);
        reinterpret_cast<uint4 *>(dst)[j] = u;
    }
}

__device__ __forceinline__ void st_global(bf16 *dst, const float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 u;
        __nv_bfloat162 *hh = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) hh[i] = __floats2bfloat162_rn(v[8 * j + 2 * i], v[8 * j + 2 * i + 1]);
        reinterpret_cast<uint4 *>(dst)[j] = u;
    }
}

__device__ __forceinline__ void st_global(float *dst, const float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4 *>(dst)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// N 64 x 64 fp32 blocks (row stride ld floats, 16-byte aligned) into fp16
// tiles, every load in flight before the first store; the whole CTA (256
// threads, 16 values each per block), no barrier.
template <int N>
__device__ __forceinline__ void tiles_from_f32(uint8_t *const (&tiles)[N], const float *const (&src)[N],
                                               const int (&ld)[N])
{
    const int t = threadIdx.x, row = t >> 2, c = (t & 3) * 16;
    float4 q[N][4];
#pragma unroll
    for (int n = 0; n < N; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[n][i] = reinterpret_cast<const float4 *>(src[n] + (long long)row * ld[n] + c)[i];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const float *f = reinterpret_cast<const float *>(q[n]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint4 u;
            __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) hh[i] = __floats2half2_rn(f[8 * j + 2 * i], f[8 * j + 2 * i + 1]);
            *reinterpret_cast<uint4 *>(tiles[n] + tc::sw128_offset(row, c + 8 * j)) = u;
        }
    }
}

// Row r, columns [c0, c0 + 32) of an fp16 tile negated in place.
__device__ __forceinline__ void negate_in_place(uint8_t *tile, int r, int c0)
{
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + tc::sw128_offset(r, c0 + 8 * j));
        uint4 u = *p;
        u.x ^= 0x80008000u, u.y ^= 0x80008000u, u.z ^= 0x80008000u, u.w ^= 0x80008000u;
        *p = u;
    }
}

// A 64 x 64 fp16 tile negated in place; the whole CTA (256 threads), no barrier.
__device__ __forceinline__ void negate_tile(uint8_t *tile)
{
    const int t = threadIdx.x, row = t >> 2, c = (t & 3) * 16;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + tc::sw128_offset(row, c + 8 * j));
        uint4 u = *p;
        u.x ^= 0x80008000u, u.y ^= 0x80008000u, u.z ^= 0x80008000u, u.w ^= 0x80008000u;
        *p = u;
    }
}

// 32 fp32 values from global memory (16-byte aligned source).
__device__ __forceinline__ void ld_global(const float *src, float (&v)[32])
{
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 f = reinterpret_cast<const float4 *>(src)[j];
        v[4 * j] = f.x;
        v[4 * j + 1] = f.y;
        v[4 * j + 2] = f.z;
        v[4 * j + 3] = f.w;
    }
}

// The inverses of the four 16 x 16 unit lower triangular diagonal blocks of
// I + A for both halves: threads 0..127, one column each (block tid / 16,
// column tid % 16), by forward substitution in fp32. sA16: [2][4][16][16] the
// strictly lower parts (entries on and above the diagonal unused). Writes
// block jb of half h at rows/columns 16 jb.. of tile dinv[h] (fp16; the rest of
// the tile is left as it is).
__device__ __forceinline__ void diag_block_inverses(const float *sA16, uint8_t *const dinv[2])
{
    const int tid = threadIdx.x;
    if (tid >= 128) return;
    const int blk = tid >> 4, j = tid & 15, h = blk >> 2, jb = blk & 3;
    const float *L = sA16 + blk * 256;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float s = i == j ? 1.f : 0.f;
#pragma unroll
        for (int k = 0; k < i; ++k) s = fmaf(-L[i * 16 + k], x[k], s);
        x[i] = s;
    }
    uint8_t *t = dinv[h];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        *reinterpret_cast<__half *>(t + tc::sw128_offset(16 * jb + i, 16 * jb + j)) = __float2half_rn(x[i]);
}

}  // namespace uttc
}  // namespace path
