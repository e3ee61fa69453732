// PaTH attention backward on tensor cores (sm_100a), head dim 128.
//
// One CTA per (128-key tile J, head): the same key-owned walk as the head-dim-64
// kernel (query blocks I = last..J+1, then the diagonal block J), with the
// adjoint of the key-side transport chain carried in the loop order:
//   Khat_{J,I+1} = Khat_{J,I} P_I^T, so Abar_I = Abar_{I+1} P_I + dS^T Qtil_I, and
//   dP_I += Abar_{I+1}^T Khat_{J,I}; after the block J+1, Abar is dKtil_J.
// At head dim 128 every operand tile is twice as wide, so each 128-query block runs
// as two 64-query sub-tiles (shared memory 227 KB, tensor memory 512 columns):
//   MMA 1: S^T = Khat_{J,I} Qtil_q^T and dP^T = V_J dO_q^T   (128 keys x 64 queries)
//   threads: P = exp(scale S + c_i - c_j - lse_i), dS = P (dP - delta_i) scale
//   MMA 2: dV += P^T dO_q;  Abar (+)= [Abar_{I+1} P_I] + dS^T Qtil_q;
//          dQtil_q = dS Khat_{J,I} (64 x 128, over the spent S^T / dP^T columns);
//          once per block: dP_I = Abar_{I+1}^T Khat_{J,I}
//   drain: dQtil_q and dP_I to the global accumulators by bulk tensor reduce-add,
//          staged as fp32 boxes in the spent P^T / dS^T buffers (32 KB: dQtil_q at
//          once, dP_I in two rounds); after the block, Abar to the operand tile
//          (fp16) or, after block J+1, to dKtil_J.
// The diagonal block takes its logits from the UT prep and hands dS to its adjoint
// (dSd), as at head dim 64. One thread issues the loads and the products; all
// threads run the softmax and the drain in sequence; every wait is bounded.
#include <type_traits>

#include "attn.cuh"
#include "attn_tc.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

constexpr int D = 128;
constexpr int NT = 256;
constexpr int QS = 64;  // queries per sub-tile
constexpr float LOG2E = 1.4426950408889634f;

struct C128 {
    static constexpr int T32 = 32768, T16 = 16384;
    static constexpr int V_OFF = 0;                 // V_J [128 keys x 128], bf16, 2 panels
    static constexpr int AB_OFF = V_OFF + T32;      // Abar operand, fp16, 2 panels
    static constexpr int KH_OFF = AB_OFF + T32;     // Khat_{J,I}, fp16, 2 panels
    static constexpr int P_OFF = KH_OFF + T32;      // P_I [d x d], fp16, 2 panels
    static constexpr int Q_OFF = P_OFF + T32;       // Qtil_q [64 x 128] fp16 x 2 buffers (2 panels each)
    static constexpr int DO_OFF = Q_OFF + 2 * T16;  // dO_q [64 x 128] bf16 x 2 buffers
    static constexpr int PT_OFF = DO_OFF + 2 * T16; // P^T [128 keys x 64 queries] bf16
    static constexpr int DS_OFF = PT_OFF + T16;     // dS^T, fp16
    static constexpr int ROW_OFF = DS_OFF + T16;    // x 2 buffers: nb[64], scale * delta[64]
    static constexpr int BAR_OFF = ROW_OFF + 2 * 512;
    static constexpr int SMEM = BAR_OFF + 128 + 1024;
    // tensor-memory columns: S^T | dP^T, then dQtil (M = 64) over them; dV, Abar, dP_I
    static constexpr uint32_t T_S = 0, T_DP = 64, T_DQ = 0, T_DV = 128, T_AB = 256, T_DPI = 384;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major operand: descriptor of K-step kk (16 columns) of a [rows x 128] tile stored as
// two 64-column panels of `panel` bytes each
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk, uint32_t panel)
{
    return desc_sw128(base + (kk >> 2) * panel + (kk & 3) * 32, 16, 1024);
}

// MN-major operand: K-step kk (16 rows) of a tile whose M/N columns come in panels of `panel` bytes
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int kk, uint32_t panel)
{
    return desc_sw128(base + kk * 2048, panel, 1024);
}

template <bool FOX, typename TO>
__global__ void __launch_bounds__(NT, 1)
    bwd128_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                     const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mDO,
                     const __grid_constant__ CUtensorMap mP, const __grid_constant__ CUtensorMap mDQ,
                     const __grid_constant__ CUtensorMap mDPI, BwdTcArgs a)
{
    using C = C128;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BAR_OFF);
    // [0] V, [1] block (Khat, P_I), [2..3] sub-tile buffers, [4] MMA, [5] the issuer's last MMAs
    uint64_t *v_full = bars, *blk_full = bars + 1, *sub_full = bars + 2, *mma_bar = bars + 4,
             *mma_done = bars + 5;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 6);
    const uint32_t s0 = smem_u32(sm);
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nblk = a.nblk, last = nblk - 1, Lp = nblk * BT;
    const int nbi = last - J + 1;  // query blocks: last..J+1, then J
    const int nsub = 2 * nbi;
    auto block_of = [&](int bi) { return bi == nbi - 1 ? J : last - bi; };

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;

    // loads (thread 0): V once, Khat / P_I per block, Qtil / dO / row terms per sub-tile
    int issued_blk = 0, issued_sub = 0;  // thread 0's count of issued block / sub-tile loads
    auto load_block = [&](int bi) {
        const int I = block_of(bi);
        const bool diag = bi == nbi - 1;
        const bool hasP = !diag && I < last;
        const uint32_t bytes = (diag ? 0 : C::T32) + (hasP ? C::T32 : 0);
        ++issued_blk;
        if (bytes == 0) {
            mbar_arrive(blk_full);  // nothing to load: complete the phase
            return;
        }
        mbar_expect_tx(blk_full, bytes);
        if (!diag) {
            const int row = (int)((h * a.npairs + (long long)I * (I - 1) / 2 + J) * BT);
            for (int p = 0; p < 2; ++p) tma_load_2d(sm + C::KH_OFF + p * C::T16, &mK, 64 * p, row, blk_full);
        }
        if (hasP)
            for (int p = 0; p < 2; ++p)
                tma_load_2d(sm + C::P_OFF + p * C::T16, &mP, 64 * p, (h * nblk + I) * D, blk_full);
    };
    auto load_sub = [&](int s) {
        const int bi = s >> 1, q = s & 1, buf = s & 1;
        const int I = block_of(bi);
        const bool diag = bi == nbi - 1;
        uint64_t *bar = &sub_full[buf];
        const int q0 = I * BT + q * QS;  // first query of the sub-tile
        ++issued_sub;
        mbar_expect_tx(bar, (diag ? 0 : C::T16) + C::T16 + 512);
        if (!diag)
            for (int p = 0; p < 2; ++p)
                tma_load_2d(sm + C::Q_OFF + buf * C::T16 + p * 8192, &mQ, 64 * p, h * Lp + q0, bar);
        for (int p = 0; p < 2; ++p)
            tma_load_3d(sm + C::DO_OFF + buf * C::T16 + p * 8192, &mDO, 64 * p, q0, h, bar);
        float *rows = reinterpret_cast<float *>(sm + C::ROW_OFF + buf * 512);
        bulk_load(rows, a.lse_p + (long long)h * Lp + q0, 256, bar);
        bulk_load(rows + 64, a.delta + (long long)h * Lp + q0, 256, bar);
    };
    if (tid == 0) {
        mbar_expect_tx(v_full, C::T32);
        for (int p = 0; p < 2; ++p) tma_load_3d(sm + C::V_OFF + p * C::T16, &mV, 64 * p, J * BT, h, v_full);
        load_block(0);
        load_sub(0);
        if (nsub > 1) load_sub(1);
    }

    // thread roles in the element-wise phases: key row j = TMEM lane, 32 columns of 64
    const int j = 32 * (warp & 3) + lane, cg = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int gj = J * BT + j;
    const float k1 = a.scale * LOG2E;
    const float cj2 = FOX ? a.c[(long long)h * Lp + gj] * LOG2E : 0.f;
    float colsum = 0.f;
    uint32_t mma_phase = 0;
    int done_blk = 0, done_sub = 0;  // block / sub-tile loads waited for (uniform)
    bool ok = mbar_wait(v_full, 0, WAIT_LIMIT_NS);
    uint8_t *sPt = sm + C::PT_OFF, *sDs = sm + C::DS_OFF;
    auto wait_mma = [&]() {
        if (ok && !mbar_wait(mma_bar, mma_phase, WAIT_LIMIT_NS)) ok = false;
        mma_phase ^= 1;
        fence_after_sync();
    };
    const uint32_t idS = idesc_f16(128, QS, AB_F16, 0, 0), idDP = idesc_f16(128, QS, AB_BF16, 0, 0);
    const uint32_t idDV = idesc_f16(128, D, AB_BF16, 0, 1), idAB = idesc_f16(128, D, AB_F16, 0, 1);
    const uint32_t idDQ = idesc_f16(QS, D, AB_F16, 1, 1), idDPI = idesc_f16(128, D, AB_F16, 1, 1);
    const uint32_t aV = s0 + C::V_OFF, aAB = s0 + C::AB_OFF, aKH = s0 + C::KH_OFF, aP = s0 + C::P_OFF;
    const uint32_t aPT = s0 + C::PT_OFF, aDS = s0 + C::DS_OFF;

#pragma unroll 1
    for (int s = 0; s < nsub; ++s) {
        const int bi = s >> 1, q = s & 1, buf = s & 1;
        const int I = block_of(bi);
        const bool diag = bi == nbi - 1;
        const bool hasP = !diag && I < last;
        const uint32_t aQ = s0 + C::Q_OFF + buf * C::T16, aDO = s0 + C::DO_OFF + buf * C::T16;
        // this sub-tile's operands (and, for its first sub-tile, the block's)
        if (ok && q == 0 && !mbar_wait(blk_full, bi & 1, WAIT_LIMIT_NS)) ok = false;
        if (ok && !mbar_wait(&sub_full[buf], (s >> 1) & 1, WAIT_LIMIT_NS)) ok = false;
        ok = __syncthreads_and(ok);
        if (ok) {
            done_blk += q == 0;
            ++done_sub;
        }
        // ---- MMA 1
        if (ok && warp == 0) {
            fence_after_sync();
            if (lane == 0) {
                if (!diag)
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tbase + C::T_S, kdesc(aKH, kk, C::T16), kdesc(aQ, kk, 8192), idS, kk > 0);
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tbase + C::T_DP, kdesc(aV, kk, C::T16), kdesc(aDO, kk, 8192), idDP, kk > 0);
                commit(mma_bar);
            }
            __syncwarp();
        }
        wait_mma();
        // ---- P, dS for 128 keys x 64 queries (this thread: key j, queries [32 cg, 32 cg + 32))
        const float *rows = reinterpret_cast<const float *>(sm + C::ROW_OFF + buf * 512);
        const float *sd = a.Sd + ((long long)h * nblk + J) * BT * BT;
        float *dsd = a.dSd + ((long long)h * nblk + J) * BT * BT;
        if (ok) {
#pragma unroll 1
            for (int c = 32 * cg; c < 32 * cg + 32; c += 16) {
                float sv[16], dp[16];
                if (diag) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) sv[u] = sd[(q * QS + c + u) * BT + j];
                } else {
                    tmem_ld16(tbase + C::T_S + c + lane_off, sv);
                }
                tmem_ld16(tbase + C::T_DP + c + lane_off, dp);
                tmem_wait_ld_tied(sv, dp);
                float pv[16], dsv[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = c + u;  // query in the sub-tile
                    const float nb = rows[i], sdl = rows[64 + i];
                    const float x = fmaf(sv[u], k1, FOX ? nb - cj2 : nb);
                    float p = ex2(x);
                    if (diag && q * QS + i < j) p = 0.f;
                    const float ds = p * fmaf(dp[u], a.scale, -sdl);
                    pv[u] = p;
                    dsv[u] = ds;
                    if (diag) dsd[(long long)(q * QS + i) * BT + j] = ds;
                }
                uint32_t pb[8], db[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const __nv_bfloat162 bb = __floats2bfloat162_rn(pv[2 * k], pv[2 * k + 1]);
                    pb[k] = *reinterpret_cast<const uint32_t *>(&bb);
                    const __half2 hh = __floats2half2_rn(dsv[2 * k], dsv[2 * k + 1]);
                    db[k] = *reinterpret_cast<const uint32_t *>(&hh);
                }
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t off = sw128_offset(j, c + 8 * hf);
                    *reinterpret_cast<uint4 *>(sPt + off) =
                        make_uint4(pb[4 * hf], pb[4 * hf + 1], pb[4 * hf + 2], pb[4 * hf + 3]);
                    *reinterpret_cast<uint4 *>(sDs + off) =
                        make_uint4(db[4 * hf], db[4 * hf + 1], db[4 * hf + 2], db[4 * hf + 3]);
                }
                if (FOX) {
                    // row (query) and column (key) sums of the fp16-rounded dS the MMAs read
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float2 f2 = __half22float2(*reinterpret_cast<const __half2 *>(&db[k]));
                        dsv[2 * k] = f2.x;
                        dsv[2 * k + 1] = f2.y;
                        colsum += f2.x + f2.y;
                    }
                    // reduce-scatter over the warp's 32 keys: lanes 2m, 2m+1 end with query c + m
#pragma unroll
                    for (int o = 16, n = 16; o >= 2; o >>= 1, n >>= 1) {
                        const bool up = lane & o;
#pragma unroll
                        for (int k = 0; k < n / 2; ++k) {
                            const float send = up ? dsv[k] : dsv[k + n / 2];
                            const float keep = up ? dsv[k + n / 2] : dsv[k];
                            dsv[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    }
                    dsv[0] += __shfl_xor_sync(0xffffffffu, dsv[0], 1);
                    if (!(lane & 1))
                        atomicAdd(a.rowsum + (long long)h * Lp + I * BT + q * QS + c + (lane >> 1),
                                  dsv[0] / a.scale);
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok);
        // ---- MMA 2
        if (ok && warp == 0) {
            fence_after_sync();
            if (lane == 0) {
                // dV += P^T dO  (K = 64 queries)
                for (int kk = 0; kk < QS / 16; ++kk)
                    mma_ss(tbase + C::T_DV, desc_sw128(aPT + kk * 32, 16, 1024), mdesc(aDO, kk, 8192), idDV,
                           (s > 0 || kk > 0));
                if (!diag) {
                    if (q == 0 && hasP) {
                        // Abar = Abar_{I+1} P_I;  dP_I = Abar_{I+1}^T Khat
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ss(tbase + C::T_AB, kdesc(aAB, kk, C::T16), mdesc(aP, kk, C::T16), idAB, kk > 0);
                        for (int kk = 0; kk < BT / 16; ++kk)
                            mma_ss(tbase + C::T_DPI, mdesc(aAB, kk, C::T16), mdesc(aKH, kk, C::T16), idDPI, kk > 0);
                    }
                    // Abar += dS^T Qtil  (K = 64 queries)
                    for (int kk = 0; kk < QS / 16; ++kk)
                        mma_ss(tbase + C::T_AB, desc_sw128(aDS + kk * 32, 16, 1024), mdesc(aQ, kk, 8192), idAB,
                               (q > 0 || hasP || kk > 0));
                    // dQtil = dS Khat  (A = dS^T read MN-major, K = 128 keys)
                    for (int kk = 0; kk < BT / 16; ++kk)
                        mma_ss(tbase + C::T_DQ, desc_sw128(aDS + kk * 2048, 8192, 1024), mdesc(aKH, kk, C::T16), idDQ,
                               kk > 0);
                }
                commit(mma_bar);
            }
            __syncwarp();
        }
        wait_mma();
        // the sub-tile's buffers are free: load the sub-tile two ahead into them
        if (ok && tid == 0 && s + 2 < nsub) load_sub(s + 2);
        // ---- drain
        if (ok && !diag) {
            // staging: the spent P^T and dS^T buffers, 32 KB of fp32 boxes of 32
            // columns (128-byte rows, 128-byte swizzle)
            uint8_t *stg = sm + C::PT_OFF;
            // dQtil of the sub-tile (M = 64: rows 16 quarter + t in lanes 32 quarter + t, t < 16;
            // the TMEM loads are warp-wide, the upper lanes' values are not used): four
            // boxes of 64 rows
            {
                const int qi = 16 * (warp & 3) + (lane & 15);
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + C::T_DQ + 64 * cg + c0 + lane_off, v);
                    if (lane < 16) {
                        uint8_t *box = stg + (2 * cg + c0 / 32) * 8192 + qi * 128;
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4 *>(box + ((k ^ (qi & 7)) << 4)) =
                                make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                    }
                }
                fence_async_smem();
                __syncthreads();
                if (tid == 0) {
                    for (int b = 0; b < 4; ++b)
                        tma_reduce_add_2d(&mDQ, 32 * b, h * Lp + I * BT + q * QS, stg + b * 8192);
                    bulk_commit();
                }
            }
            if (q == 0 && hasP) {
                // dP_I rows f = j (lane), columns [64 cg, 64 cg + 64): in two rounds (one
                // per column half) of two boxes of 128 rows, once the staging is read
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    if (tid == 0) bulk_wait_read<0>();
                    __syncthreads();
                    if (cg == half) {
#pragma unroll
                        for (int c0 = 0; c0 < 64; c0 += 32) {
                            float v[32];
                            tmem_ld32(tbase + C::T_DPI + 64 * cg + c0 + lane_off, v);
                            uint8_t *box = stg + (c0 / 32) * 16384 + j * 128;
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                *reinterpret_cast<float4 *>(box + ((k ^ (j & 7)) << 4)) =
                                    make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                        }
                    }
                    fence_async_smem();
                    __syncthreads();
                    if (tid == 0) {
                        for (int b = 0; b < 2; ++b)
                            tma_reduce_add_2d(&mDPI, 64 * half + 32 * b, (h * nblk + I) * D, stg + b * 16384);
                        bulk_commit();
                    }
                }
            }
            if (q == 1) {
                // Abar_I: the next block's operand, or dKtil_J after the block J + 1
#pragma unroll 1
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + C::T_AB + 64 * cg + c0 + lane_off, v);
                    if (I > J + 1) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            uint4 u;
                            __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                            for (int k = 0; k < 4; ++k) hh[k] = __floats2half2_rn(v[8 * g + 2 * k], v[8 * g + 2 * k + 1]);
                            *reinterpret_cast<uint4 *>(sm + C::AB_OFF + cg * C::T16 + sw128_offset(j, c0 + 8 * g)) = u;
                        }
                    } else {
                        float *dk = a.dKt + ((long long)h * Lp + gj) * D + 64 * cg + c0;
#pragma unroll
                        for (int u = 0; u < 32; u += 4)
                            *reinterpret_cast<float4 *>(dk + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
                    }
                }
            }
        }
        // the next sub-tile's softmax writes P^T and dS^T: the staging's reads end first
        if (tid == 0) bulk_wait_read<0>();
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok);
        // the block's Khat and P_I are free after its second sub-tile: load the next block's
        if (ok && tid == 0 && q == 1 && bi + 1 < nbi) load_block(bi + 1);
    }
    // the last tile has no off-diagonal pairs: its dKtil is zero
    if (ok && J == last) {
        float *dk = a.dKt + ((long long)h * Lp + gj) * D + 64 * cg;
        for (int e = 0; e < 64; e += 4) *reinterpret_cast<float4 *>(dk + e) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (ok) {
        TO *dst = static_cast<TO *>(a.dv) + ((long long)h * a.L + gj) * D + 64 * cg;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
            float v[32];
            tmem_ld32(tbase + C::T_DV + 64 * cg + c0 + lane_off, v);
            if (gj < a.L) {
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[c0 + e] = from_f<TO>(v[e]);
            }
        }
        // column sums of the gate gradient: both column halves of a key row add
        if (FOX) {
            float *cs = reinterpret_cast<float *>(sm + C::PT_OFF);  // P^T tile is free now
            if (cg == 1) cs[j] = colsum;
            __syncthreads();
            if (cg == 0 && a.colsum && gj < a.L) a.colsum[(long long)h * Lp + gj] = (colsum + cs[j]) / a.scale;
        }
    } else if (tid == 0 && a.err) {
        atomicCAS(a.err, 0, 15);
    }
    if (tid == 0) {
        // never leave with copies into this CTA's shared memory or products into its
        // tensor memory in flight (on the normal path every one was waited for)
        for (int b = done_blk; b < issued_blk; ++b) mbar_wait(blk_full, b & 1, 8 * WAIT_LIMIT_NS);
        for (int t = done_sub; t < issued_sub; ++t) mbar_wait(&sub_full[t & 1], (t >> 1) & 1, 8 * WAIT_LIMIT_NS);
        commit(mma_done);
        mbar_wait(mma_done, 0, 8 * WAIT_LIMIT_NS);
        bulk_wait_all();  // and every reduction from the staging has completed
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <bool FOX, typename TO>
cudaError_t launch(const CUtensorMap *m, const BwdTcArgs &a, cudaStream_t st)
{
    auto k = bwd128_tc_kernel<FOX, TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C128::SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nblk, a.nh), NT, C128::SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], a);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool attn_bwd128_tc_supported(Types t, int d) { return t.in == BF16 && t.mid == F16 && d == 128; }

cudaError_t attn_bwd128_tc(const BwdArgs &b, Types t, float *lse_p, void *dout_bf16, int *err,
                           cudaStream_t st)
{
    const int Lp = b.nblk * BT;
    const long long npairs = (long long)b.nblk * (b.nblk - 1) / 2;
    const void *dob = t.out == F32 ? dout_bf16 : b.dout;
    CUtensorMap m[7];
    if (!make_map_2d(&m[0], b.Qt, F16, D, (uint64_t)b.nh * Lp, QS)) return cudaErrorInvalidValue;
    if (npairs > 0) {
        if (!make_map_2d(&m[1], b.Khat, F16, D, (uint64_t)b.nh * npairs * BT, BT)) return cudaErrorInvalidValue;
    } else {
        m[1] = m[0];
    }
    if (!make_map_3d(&m[2], b.v, BF16, D, b.L, b.nh, BT) ||
        !make_map_3d(&m[3], dob, BF16, D, b.L, b.nh, QS) ||
        !make_map_2d(&m[4], b.Pm, F16, D, (uint64_t)b.nh * b.nblk * D, D) ||
        !make_map_f32_2d(&m[5], b.dQt, D, (uint64_t)b.nh * Lp, QS) ||
        !make_map_f32_2d(&m[6], b.dPm, D, (uint64_t)b.nh * b.nblk * D, D))
        return cudaErrorInvalidValue;
    BwdTcArgs a{b.Sd, b.c, lse_p, b.delta, b.scale, b.L, b.nblk, b.nh, npairs,
                b.dQt, b.dKt, b.dPm, b.dSd, b.dv, b.rowsum, b.colsum, err};
    const bool fox = b.c != nullptr;
    if (t.out == F32) return fox ? launch<true, float>(m, a, st) : launch<false, float>(m, a, st);
    return fox ? launch<true, bf16>(m, a, st) : launch<false, bf16>(m, a, st);
}

}  // namespace path
