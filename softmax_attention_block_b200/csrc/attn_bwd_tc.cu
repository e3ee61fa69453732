// PaTH attention backward on tensor cores (sm_100a), head dim 64.
//
// One CTA per (128-key tile J, head), walking the query tiles I = last..J+1,
// then the diagonal tile I = J. Keys are the CTA's rows: TMEM lane j is key j
// for S^T, dP^T, dV and the chain adjoint Abar. Per tile pair:
//   MMA 1:  S^T  = Khat_{J,I} Qtil_I^T          (fp16)
//           dP^T = V_J dO_I^T                    (bf16)
//   threads: P = exp(scale S + c_i - c_j - lse_i), dZ = P (dP - delta_i),
//            dS = scale dZ; P^T (bf16) and dS^T (fp16) to shared memory
//   MMA 2:  dV   += P^T dO_I                              (bf16)
//           dP_I += Abar_{I+1}^T Khat_{J,I}                (fp16; operand
//                   [Abar | Khat] so the M=128 form applies, top half kept)
//           Abar  = Abar_{I+1} P_I + dS^T Qtil_I           (fp16, fp32 in TMEM)
//           dQtil_I += dS Khat_{J,I}                       (fp16)
//           [gate] row sums of dS                          (dS times a ones column)
// Khat_{J,I+1} = Khat_{J,I} P_I^T, so Abar is the adjoint carried back along
// the key-side transport chain; after the pair (J+1, J) it is dKtil_J. dQtil,
// dP and the row sums accumulate across CTAs with fp32 vector reductions.
// The diagonal tile takes its logits from the UT prep and writes dS to the
// prep's adjoint instead (dSd), which carries it to dQ, dK, dW, dbeta.
#include "attn.cuh"
#include "attn_tc.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

constexpr int D = 64;
constexpr int NT = 192;
constexpr int W_PROD = 4, W_MMA = 5;
constexpr float LOG2E = 1.4426950408889634f;

struct BCfg {
    static constexpr int TILE = 128 * D * 2;     // 16 KB
    static constexpr int AB_OFF = 0;             // Abar operand (fp16), before the stages
    static constexpr int V_OFF = AB_OFF + TILE;
    static constexpr int PT_OFF = V_OFF + TILE;  // P^T  [keys x queries] bf16, 2 panels
    static constexpr int DS_OFF = PT_OFF + 2 * 16384;  // dS^T [keys x queries] fp16
    static constexpr int ONE_OFF = DS_OFF + 2 * 16384; // ones [16 x 128] fp16, 2 panels of 2 KB
    static constexpr int ST_OFF = ONE_OFF + 4096;
    // stage: Khat, Qtil, dO, P_I (8 KB), rows (lse, delta, c: 3 x 512 B)
    static constexpr int S_KH = 0, S_Q = TILE, S_DO = 2 * TILE, S_P = 3 * TILE, S_ROW = 3 * TILE + 8192;
    static constexpr int ST_BYTES = 3 * TILE + 8192 + 2048;
    static constexpr int BAR_OFF = ST_OFF + 2 * ST_BYTES;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    // TMEM columns
    static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_AB = 320;
    static constexpr uint32_t T_DQ = 0, T_RS = 64, T_DPI = 128;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void red_add_v4(float *dst, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

template <bool FOX, typename TO>
__global__ void __launch_bounds__(NT, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                  const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mDO,
                  const __grid_constant__ CUtensorMap mP, BwdTcArgs a)
{
    using C = BCfg;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    uint8_t *sAb = sm + C::AB_OFF, *sV = sm + C::V_OFF, *sPt = sm + C::PT_OFF, *sDs = sm + C::DS_OFF;
    uint8_t *sOne = sm + C::ONE_OFF;
    auto stage = [&](int s) { return sm + C::ST_OFF + s * C::ST_BYTES; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BAR_OFF);
    uint64_t *v_full = bars, *ld_full = bars + 1, *ld_empty = bars + 3, *s_full = bars + 5,
             *p_full = bars + 6, *m2_full = bars + 7, *e_done = bars + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 9);

    const int J = blockIdx.x, h = blockIdx.y;
    const int nblk = a.nblk, last = nblk - 1, Lp = nblk * BT;
    const int niter = last - J + 1;  // off-diagonal tiles last..J+1, then the diagonal
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, tid = threadIdx.x;
    auto tile_of = [&](int it) { return it == niter - 1 ? J : last - it; };

    if (tid == 0) {
        mbar_init(v_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ld_full[s], 1);
            mbar_init(&ld_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(m2_full, 1);
        mbar_init(e_done, 128);
        mbar_fence_init();
    }
    // ones column for the row sums of dS: B operand [16 x 128 keys], row 0 = 1
    for (int e = tid; e < 16 * 128; e += NT) {
        const int n = e / 128, k = e % 128;
        *reinterpret_cast<f16 *>(sOne + (k >> 6) * 2048 + sw128_offset(n, k & 63)) =
            __float2half_rn(n == 0 ? 1.f : 0.f);
    }
    fence_async_smem();
    if (warp == W_MMA) tmem_alloc(tmem_slot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_expect_tx(v_full, C::TILE);
            tma_load_3d(sV, &mV, 0, J * BT, h, v_full);
            int issued = 0;
            for (int it = 0; it < niter; ++it) {
                const int s = it & 1;
                if (it >= 2 && !mbar_wait(&ld_empty[s], ((it >> 1) - 1) & 1, WAIT_POLLS)) {
                    if (a.err) atomicCAS(a.err, 0, 11);
                    break;
                }
                const int I = tile_of(it);
                const bool diag = it == niter - 1;
                const bool hasP = !diag && I < last;
                uint8_t *st = stage(s);
                const uint32_t bytes = C::TILE * (diag ? 1 : 3) + (hasP ? 8192 : 0) + 1536;
                mbar_expect_tx(&ld_full[s], bytes);
                if (!diag) {
                    const int row = (int)((h * a.npairs + (long long)I * (I - 1) / 2 + J) * BT);
                    tma_load_2d(st + C::S_KH, &mK, 0, row, &ld_full[s]);
                    tma_load_2d(st + C::S_Q, &mQ, 0, h * Lp + I * BT, &ld_full[s]);
                }
                tma_load_3d(st + C::S_DO, &mDO, 0, I * BT, h, &ld_full[s]);
                if (hasP) tma_load_2d(st + C::S_P, &mP, 0, (h * nblk + I) * D, &ld_full[s]);
                float *rows = reinterpret_cast<float *>(st + C::S_ROW);
                bulk_load(rows, a.lse_p + (long long)h * Lp + I * BT, 512, &ld_full[s]);
                bulk_load(rows + 128, a.delta + (long long)h * Lp + I * BT, 512, &ld_full[s]);
                bulk_load(rows + 256, a.c ? a.c + (long long)h * Lp + I * BT : a.delta, 512, &ld_full[s]);
                issued = it + 1;
            }
            for (int it = issued - 2 > 0 ? issued - 2 : 0; it < issued; ++it)
                mbar_wait(&ld_full[it & 1], (it >> 1) & 1, WAIT_POLLS);
        }
    } else if (warp == W_MMA) {
        if (lane == 0) {
            const uint32_t idS = idesc_f16(128, 128, AB_F16, 0, 0);
            const uint32_t idDP = idesc_f16(128, 128, AB_BF16, 0, 0);
            const uint32_t idDV = idesc_f16(128, D, AB_BF16, 0, 1);
            const uint32_t idAbP = idesc_f16(128, D, AB_F16, 0, 1);
            const uint32_t idMN = idesc_f16(128, D, AB_F16, 1, 1);
            const uint32_t idRS = idesc_f16(128, 16, AB_F16, 1, 0);
            const uint32_t ab0 = smem_u32(sAb), v0 = smem_u32(sV), pt0 = smem_u32(sPt),
                           ds0 = smem_u32(sDs), one0 = smem_u32(sOne);
            bool ok = mbar_wait(v_full, 0, WAIT_POLLS);
            for (int it = 0; ok && it < niter; ++it) {
                const int s = it & 1, I = tile_of(it);
                const bool diag = it == niter - 1;
                if (!mbar_wait(&ld_full[s], (it >> 1) & 1, WAIT_POLLS) ||
                    (it >= 1 && !mbar_wait(e_done, (it - 1) & 1, WAIT_POLLS))) {
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t kh0 = smem_u32(stage(s) + C::S_KH), q0 = smem_u32(stage(s) + C::S_Q),
                               do0 = smem_u32(stage(s) + C::S_DO), p0 = smem_u32(stage(s) + C::S_P);
                // MMA 1
                if (!diag) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tbase + C::T_S, desc_sw128(kh0 + kk * 32, 16, 1024),
                               desc_sw128(q0 + kk * 32, 16, 1024), idS, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tbase + C::T_DP, desc_sw128(v0 + kk * 32, 16, 1024),
                           desc_sw128(do0 + kk * 32, 16, 1024), idDP, kk > 0);
                commit(s_full);
                if (!mbar_wait(p_full, it & 1, WAIT_POLLS)) {
                    ok = false;
                    break;
                }
                fence_after_sync();
                // MMA 2: dV += P^T dO   (K = 128 queries)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tbase + C::T_DV, desc_sw128(pt0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                           desc_sw128(do0 + kk * 2048, 16384, 1024), idDV, (it > 0 || kk > 0));
                if (!diag) {
                    if (I < last) {
                        // dP_I (+)= [Abar | Khat]^T Khat  (rows 0..63 = Abar^T Khat)
                        const uint32_t lbo = kh0 - ab0;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tbase + C::T_DPI, desc_sw128(ab0 + kk * 2048, lbo, 1024),
                                   desc_sw128(kh0 + kk * 2048, 16384, 1024), idMN, kk > 0);
                        // Abar = Abar_{I+1} P_I
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ss(tbase + C::T_AB, desc_sw128(ab0 + kk * 32, 16, 1024),
                                   desc_sw128(p0 + kk * 2048, 16384, 1024), idAbP, kk > 0);
                    }
                    // Abar += dS^T Qtil   (K = 128 queries)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tbase + C::T_AB, desc_sw128(ds0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                               desc_sw128(q0 + kk * 2048, 16384, 1024), idAbP, (I < last || kk > 0));
                    // dQtil = dS Khat   (A = dS^T read MN-major, K = 128 keys)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tbase + C::T_DQ, desc_sw128(ds0 + kk * 2048, 16384, 1024),
                               desc_sw128(kh0 + kk * 2048, 16384, 1024), idMN, kk > 0);
                }
                if (FOX) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tbase + C::T_RS, desc_sw128(ds0 + kk * 2048, 16384, 1024),
                               desc_sw128(one0 + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024), idRS, kk > 0);
                }
                commit(m2_full);
                commit(&ld_empty[s]);
            }
            if (!ok && a.err) atomicCAS(a.err, 0, 12);
        }
    } else {
        // elementwise warps: thread j owns key row j of tile J
        const int j = tid;
        const int gj = J * BT + j;
        const bool valid = gj < a.L;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float k1 = a.scale * LOG2E;
        const float cj2 = FOX ? a.c[(long long)h * Lp + gj] * LOG2E : 0.f;
        float colsum = 0.f;
        bool ok = true;
        for (int it = 0; it < niter; ++it) {
            const int s = it & 1, I = tile_of(it);
            const bool diag = it == niter - 1;
            if (!mbar_wait(&ld_full[s], (it >> 1) & 1, WAIT_POLLS) ||
                !mbar_wait(s_full, it & 1, WAIT_POLLS)) {
                ok = false;
                break;
            }
            fence_after_sync();
            const float *rows = reinterpret_cast<const float *>(stage(s) + C::S_ROW);
            const float *sd = a.Sd + ((long long)h * nblk + J) * BT * BT;
            float *dsd = a.dSd + ((long long)h * nblk + J) * BT * BT;
#pragma unroll 1
            for (int c0 = 0; c0 < BT; c0 += 32) {
                float sv[32], dp[32];
                if (!diag) tmem_ld32(tbase + C::T_S + c0 + lane_off, sv);
                tmem_ld32(tbase + C::T_DP + c0 + lane_off, dp);
                tmem_wait_ld();
                if (diag) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) sv[u] = sd[(c0 + u) * BT + j];
                }
                float pv[32], dsv[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int i = c0 + u;
                    const float lse2 = rows[i] * LOG2E;
                    const float bias = FOX ? rows[256 + i] * LOG2E - cj2 : 0.f;
                    float p = ex2(fmaf(sv[u], k1, bias) - lse2);
                    if (diag && i < j) p = 0.f;
                    const float dz = p * (dp[u] - rows[128 + i]);
                    pv[u] = p;
                    dsv[u] = a.scale * dz;
                    // column sums from the same fp16 values the row-sum MMA adds up, so
                    // the gate gradient's crossing sums cancel exactly
                    if (FOX) colsum += __half2float(__float2half_rn(dsv[u]));
                    if (diag) dsd[(long long)i * BT + j] = dsv[u];
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint4 up, ud;
                    __nv_bfloat162 *hp = reinterpret_cast<__nv_bfloat162 *>(&up);
                    __half2 *hd = reinterpret_cast<__half2 *>(&ud);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        hp[k] = __floats2bfloat162_rn(pv[g * 8 + 2 * k], pv[g * 8 + 2 * k + 1]);
                        hd[k] = __floats2half2_rn(dsv[g * 8 + 2 * k], dsv[g * 8 + 2 * k + 1]);
                    }
                    const int col = c0 + g * 8;
                    const uint32_t off = (col >> 6) * 16384 + sw128_offset(j, col & 63);
                    *reinterpret_cast<uint4 *>(sPt + off) = up;
                    *reinterpret_cast<uint4 *>(sDs + off) = ud;
                }
            }
            fence_async_smem();
            fence_before_sync();
            mbar_arrive(p_full);
            if (!mbar_wait(m2_full, it & 1, WAIT_POLLS)) {
                ok = false;
                break;
            }
            fence_after_sync();
            if (!diag) {
                // chain adjoint: operand for the next pair, or dKtil_J after pair (J+1, J)
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + C::T_AB + c0 + lane_off, v);
                    tmem_wait_ld();
                    if (I > J + 1) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint4 u;
                            __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                            for (int k = 0; k < 4; ++k) hh[k] = __floats2half2_rn(v[g * 8 + 2 * k], v[g * 8 + 2 * k + 1]);
                            *reinterpret_cast<uint4 *>(sAb + sw128_offset(j, c0 + g * 8)) = u;
                        }
                    } else {
                        float *dk = a.dKt + ((long long)h * Lp + gj) * D + c0;
#pragma unroll
                        for (int u = 0; u < 32; u += 4)
                            *reinterpret_cast<float4 *>(dk + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
                    }
                }
                // dQtil rows of tile I (lane = query row)
                float *dq = a.dQt + ((long long)h * Lp + I * BT + tid) * D;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + C::T_DQ + c0 + lane_off, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; u += 4) red_add_v4(dq + c0 + u, v[u], v[u + 1], v[u + 2], v[u + 3]);
                }
                if (I < last) {
                    // dP_I rows f = 0..63 live in lanes 0..63 (warps 0, 1)
                    float v[32];
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        tmem_ld32(tbase + C::T_DPI + c0 + lane_off, v);
                        tmem_wait_ld();
                        if (tid < D) {
                            float *dpm = a.dPm + (((long long)h * nblk + I) * D + tid) * D + c0;
#pragma unroll
                            for (int u = 0; u < 32; u += 4) red_add_v4(dpm + u, v[u], v[u + 1], v[u + 2], v[u + 3]);
                        }
                    }
                }
            }
            if (FOX) {
                float v[32];
                tmem_ld32(tbase + C::T_RS + lane_off, v);
                tmem_wait_ld();
                atomicAdd(a.rowsum + (long long)h * Lp + I * BT + tid, v[0] / a.scale);
            }
            fence_before_sync();
            mbar_arrive(e_done);
        }
        // the last tile has no off-diagonal pairs: its dKtil is zero
        if (ok && J == last) {
            float *dk = a.dKt + ((long long)h * Lp + gj) * D;
            for (int e = 0; e < D; e += 4) *reinterpret_cast<float4 *>(dk + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // dV_J
        if (ok) {
            float dv[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                float v[32];
                tmem_ld32(tbase + C::T_DV + c0 + lane_off, v);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) dv[c0 + u] = v[u];
            }
            if (valid) {
                TO *dst = static_cast<TO *>(a.dv) + ((long long)h * a.L + gj) * D;
#pragma unroll
                for (int e = 0; e < D; ++e) dst[e] = from_f<TO>(dv[e]);
                if (a.colsum) a.colsum[(long long)h * Lp + gj] = colsum / a.scale;
            }
        } else if (a.err) {
            atomicCAS(a.err, 0, 13);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == W_MMA) tmem_dealloc(tbase, 512);
}

// padded lse for the tensor-core backward: rows past L get +inf (probability 0)
__global__ void pad_lse_kernel(const float *lse, float *lse_p, int L, int Lp, int nh)
{
    const long long n = (long long)nh * Lp;
    for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < n;
         x += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(x / Lp), i = (int)(x % Lp);
        lse_p[x] = i < L ? lse[(long long)h * L + i] : INFINITY;
    }
}

// bf16 copy of an fp32 tensor (the dO operand when out/dout are fp32)
__global__ void f32_to_bf16_kernel(const float *src, bf16 *dst, long long n)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

template <bool FOX, typename TO>
cudaError_t launch(const CUtensorMap *m, const BwdTcArgs &a, cudaStream_t st)
{
    auto k = bwd_tc_kernel<FOX, TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg::SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nblk, a.nh), NT, BCfg::SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], a);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool attn_bwd_tc_supported(Types t, int d) { return t.in == BF16 && t.mid == F16 && d == 64; }

cudaError_t attn_bwd_tc(const BwdArgs &b, Types t, float *lse_p, void *dout_bf16, int *err,
                        cudaStream_t st)
{
    const int Lp = b.nblk * BT;
    const long long npairs = (long long)b.nblk * (b.nblk - 1) / 2;
    pad_lse_kernel<<<592, 256, 0, st>>>(b.lse, lse_p, b.L, Lp, b.nh);
    count_launches();
    const void *dob = b.dout;
    if (t.out == F32) {
        const long long n = (long long)b.nh * b.L * D;
        f32_to_bf16_kernel<<<1184, 256, 0, st>>>(static_cast<const float *>(b.dout),
                                                 static_cast<bf16 *>(dout_bf16), n);
        count_launches();
        dob = dout_bf16;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap m[5];
    if (!make_map_2d(&m[0], b.Qt, F16, D, (uint64_t)b.nh * Lp, 128)) return cudaErrorInvalidValue;
    if (npairs > 0) {
        if (!make_map_2d(&m[1], b.Khat, F16, D, (uint64_t)b.nh * npairs * BT, 128)) return cudaErrorInvalidValue;
    } else {
        m[1] = m[0];
    }
    if (!make_map_3d(&m[2], b.v, BF16, D, b.L, b.nh, 128) ||
        !make_map_3d(&m[3], dob, BF16, D, b.L, b.nh, 128) ||
        !make_map_2d(&m[4], b.Pm, F16, D, (uint64_t)b.nh * b.nblk * D, D))
        return cudaErrorInvalidValue;
    BwdTcArgs a{b.Sd, b.c, lse_p, b.delta, b.scale, b.L, b.nblk, b.nh, npairs,
                b.dQt, b.dKt, b.dPm, b.dSd, b.dv, b.rowsum, b.colsum, err};
    const bool fox = b.c != nullptr;
    if (t.out == F32) return fox ? launch<true, float>(m, a, st) : launch<false, float>(m, a, st);
    return fox ? launch<true, bf16>(m, a, st) : launch<false, bf16>(m, a, st);
}

}  // namespace path
