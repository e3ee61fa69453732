// Batched small GEMM of the closed-form UT transform on 5th-generation tensor
// cores (tcgen05, kind::tf32): the same contract as gemm_batched (GemmArgs),
// for bf16 inputs at the head dims without per-half UT kernels (16, 32).
// Products are split TF32: each operand is staged as hi (rounded to TF32) and
// lo (the fp32 remainder), and every K step adds hi.hi + hi.lo + lo.hi, so the
// products hold about 21 significant bits. One TF32 pass was measured too
// coarse for the closed form of a 128-position block at head dim 128, when that
// head dim still ran here (the fp32-output gradient error of dw tripled). fp32
// inputs keep the CUDA-core gemm_batched.
//
// One CTA of 256 threads per batch item (head, block), three CTAs per SM: C
// [M x N] with M, N, K <= 128. Per term and 32-wide quarter of K the operands are staged in shared
// memory as fp32 K-major 128-byte-swizzled panels of 32 K-values (A: M rows
// padded to 128, B: N rows), masks, the sequence limit and alpha applied while
// staging; one thread issues the MMAs into a tensor-memory accumulator shared
// by the terms. The epilogue reads the accumulator row by row (thread = row)
// and applies the row scale, the addend, the identity and the output mask.
#include "common.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

constexpr int NT = 256;
constexpr int RP = 128;                    // rows of a staged operand (padded)
constexpr int PANEL = RP * 128;            // bytes of one 32-wide K panel
constexpr int KH = 32;                     // K staged per round
constexpr int OPB = PANEL;                 // bytes of one staged operand part (32 K values)
constexpr int SMEM = 4 * OPB + 1024 + 64;  // A hi / lo, B hi / lo, alignment slack, barrier + TMEM slot

// Instruction descriptor of tcgen05.mma kind::tf32 (fp32 accumulation, both
// operands K-major).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N)
{
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, tf32 operands (one thread issues)
__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// byte offset of (row r, k) in a staged operand
__device__ __forceinline__ uint32_t kmaj_offset(int r, int k)
{
    return (uint32_t)(k >> 5) * PANEL + (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128 +
           (uint32_t)((((k & 31) >> 2) ^ (r & 7)) << 4) + (uint32_t)(k & 3) * 4;
}

// x = hi + lo: hi rounded to the nearest TF32 value, lo the exact fp32 remainder
// (read by the tensor cores to TF32 again, about 2^-22 of x)
__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo)
{
    const uint32_t u = (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
    hi = (x == x && fabsf(x) < 3.0e38f) ? __uint_as_float(u) : x;
    lo = x - hi;
}

// 4 consecutive stored elements (row sr, columns sc..sc+3) as fp32
__device__ __forceinline__ void load4(const Operand &o, long long base, int sr, int sc, float (&v)[4])
{
    const long long i = base + (long long)sr * o.ld + sc;
    if (o.dt == F32) {
        const float4 f = *reinterpret_cast<const float4 *>(static_cast<const float *>(o.p) + i);
        v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
    } else if (o.dt == BF16) {
        const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const bf16 *>(o.p) + i);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        v[0] = a.x, v[1] = a.y, v[2] = b.x, v[3] = b.y;
    } else {
        const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const f16 *>(o.p) + i);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
        v[0] = a.x, v[1] = a.y, v[2] = b.x, v[3] = b.y;
    }
}

// 4 consecutive stored elements at index i (16-byte or 8-byte aligned)
template <int DT>
__device__ __forceinline__ void ld4(const void *p, long long i, float (&v)[4])
{
    if (DT == F32) {
        const float4 f = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
        v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
    } else {
        const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p) + i);
        float2 a, b;
        if (DT == BF16) {
            a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
            b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        } else {
            a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
            b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
        }
        v[0] = a.x, v[1] = a.y, v[2] = b.x, v[3] = b.y;
    }
}

template <int DT>
__device__ __forceinline__ float ld1(const void *p, long long i)
{
    if (DT == F32) return static_cast<const float *>(p)[i];
    if (DT == BF16) return __bfloat162float(static_cast<const bf16 *>(p)[i]);
    return __half2float(static_cast<const f16 *>(p)[i]);
}

// One operand of a staging round: op(X) restricted to K in [kb, kb + 4 kg) as
// an [R x 4 kg] K-major operand, hi and lo parts (kg = 1 << kglog, at least 4).
// Logical element (r, k) is stored at (r, k) (KMAJ: the stored matrix is
// [R x K]) or (k, r) (the stored matrix is [K x R]). Padding up to RP rows and
// 4 kg columns is written as zero. Every thread writes whole 16-byte chunks (4
// consecutive k of one row r); each warp covers the 8 swizzle positions of its
// rows evenly; each thread's loads are all in flight before its stores.
// EXACT: 16-bit values times alpha = +-1 are TF32 values: no lo part is staged
// (the products that would read it are not issued)
template <bool KMAJ, int DT, bool EXACT>
__device__ void stage1(const Operand &o, long long base, int R, float alpha, uint8_t *hi, uint8_t *lo,
                       int blk, int K, int kb, int kglog)
{
    constexpr int BATCH = 4;
    const int nch = RP << kglog;  // chunks to write
    const int seq_rows = o.seq >= 0 ? o.seq - blk * BT : 1 << 30;  // stored rows below this are live
    const int mask = o.mask, ld = o.ld;
    const void *p = o.p;
    for (int e0 = threadIdx.x; e0 < nch; e0 += NT * BATCH) {
        float v[BATCH][4];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int e = e0 + b * NT;
            int r, g;
            if (KMAJ) {
                // stored [R x K]: a warp takes one row's K groups in order
                r = e >> kglog, g = e & ((1 << kglog) - 1);
            } else {
                // stored [K x R]: a warp takes 8 consecutive rows r and 4 K groups,
                // each 8 threads reading 8 consecutive stored columns
                const int t = e & 31, w = e >> 5;
                r = ((w & 15) << 3) + (t & 7), g = ((w >> 4) << 2) + (t >> 3);
            }
            const int k0 = kb + 4 * g;
#pragma unroll
            for (int u = 0; u < 4; ++u) v[b][u] = 0.f;
            if (e < nch && r < R && k0 < K) {
                if (KMAJ) {
                    if (r < seq_rows) ld4<DT>(p, base + (long long)r * ld + k0, v[b]);
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (k0 + u < seq_rows) v[b][u] = ld1<DT>(p, base + (long long)(k0 + u) * ld + r);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int e = e0 + b * NT;
            if (e >= nch) break;
            int r, g;
            if (KMAJ) {
                r = e >> kglog, g = e & ((1 << kglog) - 1);
            } else {
                const int t = e & 31, w = e >> 5;
                r = ((w & 15) << 3) + (t & 7), g = ((w >> 4) << 2) + (t >> 3);
            }
            const int k0 = kb + 4 * g;
            float h4[4], l4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                // masks act on stored (row, column)
                const int sr = KMAJ ? r : k0 + u, sc = KMAJ ? k0 + u : r;
                const bool z = (mask == MASK_LOWER && sc > sr) || (mask == MASK_STRICT_LOWER && sc >= sr);
                if (EXACT)
                    h4[u] = z ? 0.f : alpha * v[b][u], l4[u] = 0.f;
                else
                    split_tf32(z ? 0.f : alpha * v[b][u], h4[u], l4[u]);
            }
            const uint32_t off = kmaj_offset(r, 4 * g);
            *reinterpret_cast<float4 *>(hi + off) = make_float4(h4[0], h4[1], h4[2], h4[3]);
            if (!EXACT) *reinterpret_cast<float4 *>(lo + off) = make_float4(l4[0], l4[1], l4[2], l4[3]);
        }
    }
}

__device__ void stage(const Operand &o, long long base, int R, bool kmaj, float alpha, uint8_t *hi,
                      uint8_t *lo, int blk, int K, int kb, int kglog)
{
    if (!o.p) {
        // no operand: zeros
        for (int i = threadIdx.x; i < (RP << kglog); i += NT) {
            const int r = i >> kglog, g = i & ((1 << kglog) - 1);
            *reinterpret_cast<float4 *>(hi + kmaj_offset(r, 4 * g)) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(lo + kmaj_offset(r, 4 * g)) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
#define STAGE_CASE(DT, EX)                                                                 \
    if (o.dt == DT) {                                                                      \
        if (kmaj)                                                                          \
            stage1<true, DT, EX>(o, base, R, alpha, hi, lo, blk, K, kb, kglog);            \
        else                                                                               \
            stage1<false, DT, EX>(o, base, R, alpha, hi, lo, blk, K, kb, kglog);           \
        return;                                                                            \
    }
    const bool unit = alpha == 1.f || alpha == -1.f;
    STAGE_CASE(F32, false)
    if (unit) {
        STAGE_CASE(BF16, true)
        STAGE_CASE(F16, true)
    } else {
        STAGE_CASE(BF16, false)
        STAGE_CASE(F16, false)
    }
#undef STAGE_CASE
}

__global__ void __launch_bounds__(NT, 3) gemm_tc_kernel(GemmArgs g)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    uint8_t *sAh = sm, *sAl = sm + OPB, *sBh = sm + 2 * OPB, *sBl = sm + 3 * OPB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 4 * OPB);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Np = (g.N + 15) & ~15;
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tslot, 128);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    const uint32_t id = idesc_tf32(128, Np);
    uint32_t phase = 0;
    bool ok = true;

    for (int z = blockIdx.x; z < g.batch; z += gridDim.x) {
        const int h = z / g.nblk, blk = z % g.nblk;
        bool first = true;
        for (int t = 0; t < g.nterms; ++t) {
            const Term &T = g.t[t];
            const long long abase = (long long)h * T.a.sh + (long long)blk * T.a.sb;
            const long long bbase = (long long)h * T.b.sh + (long long)blk * T.b.sb;
            for (int kb = 0; kb < g.K; kb += KH) {
                const int kspan = g.K - kb < KH ? g.K - kb : KH;
                const int kglog = kspan == 32 ? 3 : 2;
                // A: logical [M x K], stored [M x K] (K-major) unless transposed
                stage(T.a, abase, g.M, !T.a.trans, T.alpha, sAh, sAl, blk, g.K, kb, kglog);
                // B: logical [K x N] staged as [N x K], stored [N x K] when transposed
                stage(T.b, bbase, g.N, T.b.trans != 0, 1.f, sBh, sBl, blk, g.K, kb, kglog);
                fence_async_smem();
                fence_before_sync();
                __syncthreads();
                if (warp == 0) {
                    fence_after_sync();
                    if (lane == 0) {
                        const uint32_t ah = smem_u32(sAh), al = smem_u32(sAl), bh = smem_u32(sBh),
                                       bl = smem_u32(sBl);
                        // operands exact in TF32 have no lo part: their lo product is not issued
                        const bool a_lo = !(T.a.dt != F32 && (T.alpha == 1.f || T.alpha == -1.f));
                        const bool b_lo = T.b.dt == F32;
                        for (int kk = 0; kk < kspan / 8; ++kk) {
                            const uint32_t off = (uint32_t)(kk >> 2) * PANEL + (uint32_t)(kk & 3) * 32;
                            // small terms first
                            if (a_lo) {
                                mma_tf32(tbase, desc_sw128(al + off, 16, 1024), desc_sw128(bh + off, 16, 1024), id,
                                         first ? 0u : 1u);
                                first = false;
                            }
                            if (b_lo) {
                                mma_tf32(tbase, desc_sw128(ah + off, 16, 1024), desc_sw128(bl + off, 16, 1024), id,
                                         first ? 0u : 1u);
                                first = false;
                            }
                            mma_tf32(tbase, desc_sw128(ah + off, 16, 1024), desc_sw128(bh + off, 16, 1024), id,
                                     first ? 0u : 1u);
                            first = false;
                        }
                        commit(bar);
                    }
                    __syncwarp();
                }
                first = false;
                // the staged operands are read once the MMAs complete
                if (ok && !mbar_wait(bar, phase, WAIT_LIMIT_NS)) ok = false;
                phase ^= 1;
                fence_after_sync();
            }
        }
        // epilogue: thread = row r (lane quarter warp % 4), 32-column chunks of half warp / 4
        const int r = (warp & 3) * 32 + lane, chalf = warp >> 2;
        const long long cbase = (long long)h * g.csh + (long long)blk * g.csb;
        const long long ebase = (long long)h * g.addend.sh + (long long)blk * g.addend.sb;
        const bool row_ok = r < g.M && !(g.c_seq >= 0 && blk * BT + r >= g.c_seq);
        float rs = 1.f;
        if (g.rowscale && r < g.M)
            rs = (g.rs_seq >= 0 && blk * BT + r >= g.rs_seq)
                     ? 0.f
                     : g.rowscale[(long long)h * g.rs_sh + (long long)blk * g.rs_sb + r];
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int nchunk = (Np + 31) / 32;  // 32-column chunks, split between the warp groups
        for (int q = chalf; q < nchunk; q += 2) {
            const int c0 = 32 * q;
            float v[32];
            tmem_ld32(tbase + lane_off + (uint32_t)c0, v);  // columns past Np are in the allocation
            if (!row_ok) continue;
            const int nv = g.N - c0 < 32 ? g.N - c0 : 32;  // a multiple of 4
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                if (j >= nv) break;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
                if (g.addend.p && !(g.addend.seq >= 0 && blk * BT + r >= g.addend.seq))
                    load4(g.addend, ebase, r, c0 + j, a4);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = c0 + j + u;
                    float x = (g.nterms ? v[j + u] * rs : 0.f) + g.gamma * a4[u];
                    if (g.add_identity && r == c) x += 1.f;
                    if ((g.outmask == MASK_LOWER && c > r) || (g.outmask == MASK_STRICT_LOWER && c >= r)) x = 0.f;
                    v[j + u] = x;
                }
                const long long o = cbase + (long long)r * g.ldc + c0 + j;
                if (g.cdt == F32) {
                    *reinterpret_cast<float4 *>(static_cast<float *>(g.c) + o) =
                        make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) store_from_f(g.c, g.cdt, o + u, v[j + u]);
                }
            }
        }
        // the next item's staging overwrites the operands and the accumulator:
        // every thread has read its row first
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
    }
    if (!ok && tid == 0 && g.err) atomicCAS(g.err, 0, 21);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

bool aligned_operand(const Operand &o)
{
    if (!o.p) return true;
    const int es = o.dt == F32 ? 4 : 2;
    // vector access of 4 elements: base, strides and leading dimension in units of 4
    return (reinterpret_cast<uintptr_t>(o.p) % (4 * es)) == 0 && o.ld % 4 == 0 && o.sh % 4 == 0 &&
           o.sb % 4 == 0;
}

}  // namespace

bool gemm_tc_supported(const GemmArgs &g)
{
    if (g.M < 1 || g.M > 128 || g.N < 1 || g.N > 128 || g.K < 1 || g.K > 128) return false;
    // K in 32-wide rounds of 16 or 32 (4-wide K groups: a power of two >= 4)
    if (g.M % 4 != 0 || g.N % 4 != 0 || (g.K != 16 && g.K != 32 && g.K != 64 && g.K != 128)) return false;
    for (int t = 0; t < g.nterms; ++t)
        if (!aligned_operand(g.t[t].a) || !aligned_operand(g.t[t].b)) return false;
    if (g.addend.p && (g.addend.trans || g.addend.mask || !aligned_operand(g.addend)))
        return false;
    if (g.cdt == F32 && (reinterpret_cast<uintptr_t>(g.c) % 16 != 0 || g.ldc % 4 != 0 || g.csh % 4 != 0 ||
                         g.csb % 4 != 0))
        return false;
    return true;
}

cudaError_t gemm_batched_tc(const GemmArgs &g, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    const int grid = g.batch < 8 * 148 ? g.batch : 8 * 148;
    gemm_tc_kernel<<<grid, NT, SMEM, stream>>>(g);
    count_launches();
    return cudaGetLastError();
}

}  // namespace path
