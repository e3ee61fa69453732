// Adjoint of the per-block UT prep on tcgen05 (tensor memory), head dim 64,
// bf16 inputs: one CTA per 128-position block, both 64-position halves side
// by side (ut_tc.cuh).
//
// The attention backward hands over, per block, the adjoints of the
// boundary-adjusted queries / keys (dQtil, dKtil: 128 rows), of the block
// product (dP) and of the block's logits (dSd). This kernel carries them to
// dq, dk, dw and dbeta:
//
// 1. It reads each half's UT transform (Paper-Notes "训练策略":
//    T^{-1} = (I + strictLower(D W W^T))^{-1} D) from what the forward prep
//    saved (prep_fwd_ut.cu): What, U, M, the inverse X = (I + A)^{-1} itself,
//    and the composition's inputs Ktil_a, Qtil_b, P_a, P_b.
// 2. The halves compose the block (Qtil[b] = Qtil_b P_a, Ktil[a] = Ktil_a P_b^T,
//    P = P_b P_a, Sd[b,a] = Qtil_b Ktil_a^T), so the block's adjoints become
//    per-half ones:
//      dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a,  dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b,
//      dP_a = Qtil_b^T dQtil[b] + P_b^T dP,          dP_b = dKtil[a]^T Ktil_a + dP P_a^T.
// 3. Per half, with Qtil = Q - M What, Ktil = K - U^T W, P = I - W^T What,
//    Sd = lower(Q K^T - M U) and adjoints dQ, dK, dP, dS:
//      dWhat = -M^T dQ - W dP,  dU = -W dK^T - M^T dS,  dM = lower(-dQ What^T - dS U^T)
//      dq = dQ + dS K + dM W
//      dR = X^T [dWhat | dU]                         (the transposed solve)
//      dA = strictLower(-(dR_w What^T + dR_n U^T)),  dN = strictLower(D dR_n), dG = strictLower(D dA)
//      dbeta_r = dR_w[r].W[r] + dR_n[r].N[r] + sum_c dA[r][c] G[r][c]    (G = W W^T)
//      dk = dK + dS^T Q + dN^T W
//      dw = D dR_w - U dK - What dP^T + dM^T Q + dN K + (dG + dG^T) W
//
// Products run on fp16 operands (the bf16 inputs are exact in fp16) with fp32
// accumulation; dq, dk, dw add the fp32 adjoints dQ, dK and D dR_w, and dbeta
// is formed from fp32 values.
#include "prep.cuh"
#include "runtime.cuh"
#include "ut_tc.cuh"

namespace path {

namespace {

using namespace tc;
using namespace uttc;

constexpr int NT = 256;
constexpr int SAVED_WORD = UT_SAVED_BYTE * 0x01010101;

// shared-memory tiles (8 KB each); "_h" = half a at the index, half b at +1
// unless noted
enum {
    T_W = 0, T_K = 1,       // W_h at 2h, K_h at 2h + 1 ([W_h; K_h] is one 128-row operand)
    T_Q = 4,                // Q_h
    T_E = 6,                // (Ktil_a, Qtil_b) -> dP_h
    T_NN = 8,               // (dQtil[b], dKtil[a]) -> dWhat_h -> dR_n_h -> dG_h
    T_Z = 10,               // per half (b at +3): What, U, X
    T_DPB = 16,             // dP (the block's)
    T_M = 17,               // M_h -> dM_h
    T_P = 19,               // (P_a, P_b) -> dU_h -> dN_h
    T_DSBA = 21,            // dSd[b, a]
    T_DQ = 22,              // dQ_h -> dR_w_h
    T_DK = 24,              // dK_h
    T_DS = 26,              // dS_h
    NTILES = 28,
};
constexpr int BETA_OFF = NTILES * TILE;
constexpr int PART_OFF = BETA_OFF + 128 * 4;  // [2][128] dbeta partial sums
constexpr int BAR_OFF = PART_OFF + 256 * 4;
constexpr int SMEM = BAR_OFF + 64 + 1024;

// tensor-memory columns
constexpr int C_CA = 128;                             // dKtil_a | dQtil_b, then dP_a | dP_b at +64
constexpr int C_B1 = 0;                               // dWhat', dU', dM' at +0, +64, +128
constexpr int C_DR = 256;                             // dR_w | dR_n (held to the end)
constexpr int C_DQ = 0;                               // dS K + dM W
constexpr int C_DA = 64, C_DKK = 128, C_GN2 = 384;    // dA', dS^T Q + dN^T W, W [W; K]^T again
constexpr int C_W1 = 0, C_W2 = 64;                    // dw: positive and negative terms

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Row r, columns [c0, c0 + 32) of a bf16 tile converted to fp16 in place.
__device__ __forceinline__ void to_f16_in_place(uint8_t *tile, int r, int c0)
{
    float v[32];
    ld_tile_bf16(tile, r, c0, v);
    st_tile_f16(tile, r, c0, v);
}

template <typename TO>
__global__ void __launch_bounds__(NT, 1)
    prep_bwd_ut_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mQ,
                       const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mH,
                       const __grid_constant__ CUtensorMap mB, const float *beta, int L, int nblk,
                       float *dQt, float *dKt, const float *dPm, const float *dSd, TO *dq, TO *dk,
                       TO *dw, float *dbeta, int nsm, const int *saved, int *err)
{
    if (*saved != SAVED_WORD) {  // nothing to read: record it, write nothing
        if (threadIdx.x == 0 && err) atomicCAS(err, 0, ERR_UT_NOT_SAVED);
        return;
    }
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    auto tile = [&](int i) { return sm + i * TILE; };
    const uint32_t s0 = smem_u32(sm);
    auto ta = [&](int i) { return s0 + (uint32_t)i * TILE; };
    float *sB = reinterpret_cast<float *>(sm + BETA_OFF);
    float *sPart = reinterpret_cast<float *>(sm + PART_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + BAR_OFF);  // [0] loads, [1] MMA
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int J = blockIdx.x, hd = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Lp = nblk * BT;
    const long long brow = (long long)hd * Lp + (long long)J * BT;  // block's first row in [nh, Lp]
    const long long blk = (long long)hd * nblk + J;
    const float *dsdb = dSd + blk * BT * BT;
    // the save area's tensor maps: mH over the per-half arrays What, U, X, M
    // ([nblk_all 2 64, 64] each, stacked in that order at stride hstride rows),
    // mB over the per-block ones Kta, Qtb, Pa, Pb ([nblk_all 64, 64], bstride rows)
    const long long nb_all = (long long)nblk * gridDim.y;
    const int hstride = (int)(nb_all * 2 * HB), bstride = (int)(nb_all * HB);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        mbar_expect_tx(&bars[0], 18 * TILE);
        for (int h = 0; h < 2; ++h) {
            const int y = J * BT + h * HB, yh = (int)(blk * 2 + h) * HB;
            tma_load_3d(tile(T_W + 2 * h), &mW, 0, y, hd, &bars[0]);
            tma_load_3d(tile(T_K + 2 * h), &mK, 0, y, hd, &bars[0]);
            tma_load_3d(tile(T_Q + h), &mQ, 0, y, hd, &bars[0]);
            for (int m = 0; m < 3; ++m)  // What, U, X
                tma_load_2d(tile(T_Z + 3 * h + m), &mH, 0, m * hstride + yh, &bars[0]);
            tma_load_2d(tile(T_M + h), &mH, 0, 3 * hstride + yh, &bars[0]);
            tma_load_2d(tile(T_E + h), &mB, 0, h * bstride + (int)blk * HB, &bars[0]);  // Ktil_a, Qtil_b
            tma_load_2d(tile(T_P + h), &mB, 0, (2 + h) * bstride + (int)blk * HB, &bars[0]);  // P_a, P_b
        }
        // one CTA per SM, started in grid order: the block nsm places further on
        // starts on an SM this wave frees; what it reads goes to L2 meanwhile
        const long long n2 = blk + nsm;
        if (n2 < nb_all) {
            const int J2 = (int)(n2 % nblk), h2 = (int)(n2 / nblk);
            for (int h = 0; h < 2; ++h) {
                tma_prefetch_3d(&mW, 0, J2 * BT + h * HB, h2);
                tma_prefetch_3d(&mK, 0, J2 * BT + h * HB, h2);
                tma_prefetch_3d(&mQ, 0, J2 * BT + h * HB, h2);
                for (int m = 0; m < 4; ++m) tma_prefetch_2d(&mH, 0, m * hstride + (int)(n2 * 2 + h) * HB);
                for (int m = 0; m < 2; ++m) tma_prefetch_2d(&mB, 0, (2 * m + h) * bstride + (int)n2 * HB);
            }
            const long long brow2 = (long long)h2 * Lp + (long long)J2 * BT;
            prefetch_l2(dQt + brow2 * HB, BT * HB * 4);
            prefetch_l2(dKt + brow2 * HB, BT * HB * 4);
            prefetch_l2(dPm + n2 * HB * HB, HB * HB * 4);
            prefetch_l2(dSd + n2 * BT * BT, BT * BT * 4);
        }
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    if (tid < BT) {
        const int p = J * BT + tid;
        sB[tid] = p < L ? beta[(long long)hd * L + p] : 0.f;
    }
    {   // the fp32 adjoints the composition adjoint reads, as fp16 operands
        uint8_t *const t[4] = {tile(T_NN), tile(T_NN + 1), tile(T_DPB), tile(T_DSBA)};
        const float *const src[4] = {dQt + (brow + HB) * HB, dKt + brow * HB, dPm + blk * HB * HB,
                                     dsdb + (long long)HB * BT};  // dQtil[b], dKtil[a], dP, dSd[b, a]
        const int ld[4] = {HB, HB, HB, BT};
        tiles_from_f32(t, src, ld);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = mbar_wait(&bars[0], 0, WAIT_LIMIT_NS);

    const Me me;
    const int h = me.h, r = me.r, c0 = 32 * me.cg;
    const float br = sB[h * HB + r];
    uint32_t phase = 0;
    auto sync_operands = [&]() {
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok);
    };
    auto wait_mma = [&]() {
        if (ok && !mbar_wait(&bars[1], phase, WAIT_LIMIT_NS)) ok = false;
        phase ^= 1;
        fence_after_sync();
    };
#define ISSUE(...)                 \
    do {                           \
        if (ok && warp == 0) {     \
            fence_after_sync();    \
            if (lane == 0) {       \
                __VA_ARGS__;       \
                commit(&bars[1]);  \
            }                      \
            __syncwarp();          \
        }                          \
    } while (0)

    float v[32], x[32];
    if (ok) {  // W, K, Q (bf16 inputs, exact in fp16) beside the fp16 operands; M from the saved -M
        to_f16_in_place(tile(T_W + 2 * h), r, c0);
        to_f16_in_place(tile(T_K + 2 * h), r, c0);
        to_f16_in_place(tile(T_Q + h), r, c0);
        negate_in_place(tile(T_M + h), r, c0);
    }
    sync_operands();

    // ---- CA: the block's adjoints to the halves'
    ISSUE({
        // a: dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b; dP_a = Qtil_b^T dQtil[b] + P_b^T dP
        mma64(dst(tbase, 0, C_CA), ta(T_NN + 1), A_N, ta(T_P + 1), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, C_CA), ta(T_DSBA), A_T, ta(T_E + 1), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, C_CA + 64), ta(T_E + 1), A_T, ta(T_NN), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, C_CA + 64), ta(T_P + 1), A_T, ta(T_DPB), B_N, 1, TILE, true);
        // b: dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a; dP_b = dKtil[a]^T Ktil_a + dP P_a^T
        mma64(dst(tbase, 1, C_CA), ta(T_NN), A_N, ta(T_P), B_T, 1, TILE, false);
        mma64(dst(tbase, 1, C_CA), ta(T_DSBA), A_N, ta(T_E), B_N, 1, TILE, true);
        mma64(dst(tbase, 1, C_CA + 64), ta(T_NN + 1), A_T, ta(T_E), B_N, 1, TILE, false);
        mma64(dst(tbase, 1, C_CA + 64), ta(T_DPB), A_N, ta(T_P), B_T, 1, TILE, true);
    });
    {   // meanwhile: the halves' own adjoints as fp16 operands
        uint8_t *const t[4] = {tile(T_DQ), tile(T_DK + 1), tile(T_DS), tile(T_DS + 1)};
        const float *const src[4] = {dQt + brow * HB, dKt + (brow + HB) * HB, dsdb,
                                     dsdb + (long long)HB * BT + HB};  // dQ_a, dK_b, dS_a, dS_b
        const int ld[4] = {HB, HB, BT, BT};
        tiles_from_f32(t, src, ld);
    }
    wait_mma();
    if (ok) {
        me.ld(tbase, C_CA, v);
        if (h == 0) {  // dK_a: operand, and the fp32 value dk adds (over dKtil[a])
            st_tile_f16(tile(T_DK), r, c0, v);
            st_global(dKt + (brow + r) * HB + c0, v);
        } else {       // dQ_b likewise (over dQtil[b])
            st_tile_f16(tile(T_DQ + 1), r, c0, v);
            st_global(dQt + (brow + HB + r) * HB + c0, v);
        }
        me.ld(tbase, C_CA + 64, v);
        st_tile_f16(tile(T_E + h), r, c0, v);  // dP_h
    }
    sync_operands();

    // ---- B1: dWhat = -(M^T dQ + W dP), dU = -(W dK^T + M^T dS), dM = lower(-(dQ What^T + dS U^T))
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const uint32_t w = ta(T_W + 2 * hh), m = ta(T_M + hh);
        mma64(dst(tbase, hh, C_B1), m, A_T, ta(T_DQ + hh), B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_B1), w, A_N, ta(T_E + hh), B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_B1 + 64), w, A_N, ta(T_DK + hh), B_T, 1, TILE, false);
        mma64(dst(tbase, hh, C_B1 + 64), m, A_T, ta(T_DS + hh), B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_B1 + 128), ta(T_DQ + hh), A_N, ta(T_Z + 3 * hh), B_T, 1, TILE, false);
        mma64(dst(tbase, hh, C_B1 + 128), ta(T_DS + hh), A_N, ta(T_Z + 3 * hh + 1), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, C_B1, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(T_NN + h), r, c0, v);  // dWhat
        me.ld(tbase, C_B1 + 64, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(T_P + h), r, c0, v);   // dU
        me.ld(tbase, C_B1 + 128, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j <= r ? -v[j] : 0.f;
        st_tile_f16(tile(T_M + h), r, c0, v);   // dM
    }
    sync_operands();

    // ---- B2: dR = X^T [dWhat | dU] (dWhat_h, dU_h are tiles T_NN + h, T_P + h), dS K + dM W
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        mma64(dst(tbase, hh, C_DR), ta(T_Z + 3 * hh + 2), A_T, ta(T_NN + hh), B_N, 2,
              (T_P - T_NN) * TILE, false);
        mma64(dst(tbase, hh, C_DQ), ta(T_DS + hh), A_N, ta(T_K + 2 * hh), B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_DQ), ta(T_M + hh), A_N, ta(T_W + 2 * hh), B_N, 1, TILE, true);
    });
    ld_global(dQt + (brow + h * HB + r) * HB + c0, x);  // in flight during the MMAs
    wait_mma();
    const long long grow = (long long)hd * L + (long long)J * BT + h * HB + r;  // row in [nh, L]
    const bool valid = J * BT + h * HB + r < L;
    if (ok) {
        me.ld(tbase, C_DR, v);
        st_tile_f16(tile(T_DQ + h), r, c0, v);   // dR_w
        me.ld(tbase, C_DR + 64, v);
        st_tile_f16(tile(T_NN + h), r, c0, v);   // dR_n
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j < r ? br * v[j] : 0.f;
        st_tile_f16(tile(T_P + h), r, c0, v);    // dN = strictLower(D dR_n)
        // dq = dQ + dS K + dM W
        me.ld(tbase, C_DQ, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += x[j];
        if (valid) st_global(dq + grow * HB + c0, v);
    }
    sync_operands();

    // ---- B3: dA' = dR_w What^T + dR_n U^T, dS^T Q + dN^T W, and G | N again
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const uint32_t w = ta(T_W + 2 * hh);
        mma64(dst(tbase, hh, C_DA), ta(T_DQ + hh), A_N, ta(T_Z + 3 * hh), B_T, 1, TILE, false);
        mma64(dst(tbase, hh, C_DA), ta(T_NN + hh), A_N, ta(T_Z + 3 * hh + 1), B_T, 1, TILE, true);
        mma64(dst(tbase, hh, C_DKK), ta(T_DS + hh), A_T, ta(T_Q + hh), B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_DKK), ta(T_P + hh), A_T, w, B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_GN2), w, A_N, w, B_T, 2, TILE, false);
    });
    float xk[32];
    ld_global(dKt + (brow + h * HB + r) * HB + c0, xk);  // in flight during the MMAs
    wait_mma();
    if (ok) {
        // dbeta_r = dR_w[r].W[r] + dR_n[r].N[r] + sum_c dA[r][c] G[r][c]
        float s = 0.f;
        me.ld(tbase, C_DR, v);
        ld_tile_f16(tile(T_W + 2 * h), r, c0, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) s = fmaf(v[j], x[j], s);
        me.ld(tbase, C_DR + 64, v);
        me.ld(tbase, C_GN2 + 64, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) s = fmaf(v[j], c0 + j < r ? x[j] : 0.f, s);
        me.ld(tbase, C_DA, v);
        me.ld(tbase, C_GN2, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float da = c0 + j < r ? -v[j] : 0.f;  // dA = strictLower(-dA')
            s = fmaf(da, x[j], s);
            v[j] = br * da;                           // dG = strictLower(D dA)
        }
        st_tile_f16(tile(T_NN + h), r, c0, v);
        sPart[me.cg * BT + h * HB + r] = s;
        // dk = dK + dS^T Q + dN^T W
        me.ld(tbase, C_DKK, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += xk[j];
        if (valid) st_global(dk + grow * HB + c0, v);
    }
    sync_operands();
    if (ok && me.cg == 0 && valid) dbeta[grow] = sPart[h * HB + r] + sPart[BT + h * HB + r];

    // ---- B4: dw = D dR_w + (dM^T Q + dN K + dG W + dG^T W) - (U dK + What dP^T)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const uint32_t w = ta(T_W + 2 * hh), g = ta(T_NN + hh);
        mma64(dst(tbase, hh, C_W1), ta(T_M + hh), A_T, ta(T_Q + hh), B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_W1), ta(T_P + hh), A_N, ta(T_K + 2 * hh), B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_W1), g, A_N, w, B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_W1), g, A_T, w, B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_W2), ta(T_Z + 3 * hh + 1), A_N, ta(T_DK + hh), B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_W2), ta(T_Z + 3 * hh), A_N, ta(T_E + hh), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, C_W1, v);
        me.ld(tbase, C_W2, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] -= x[j];
        me.ld(tbase, C_DR, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = fmaf(br, x[j], v[j]);
        if (valid) st_global(dw + grow * HB + c0, v);
    }
#undef ISSUE
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 22);
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <typename TO>
cudaError_t launch(const CUtensorMap *m, const PrepDims &Dm, const PrepInputs &in,
                   const PrepGrads &g, const int *saved, int *err, cudaStream_t st)
{
    auto k = prep_bwd_ut_kernel<TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(Dm.nblk, Dm.nh), NT, SMEM, st>>>(
        m[0], m[1], m[2], m[3], m[4], in.beta, Dm.L, Dm.nblk, const_cast<float *>(g.dQt),
        const_cast<float *>(g.dKt), g.dPm, g.dSd, static_cast<TO *>(g.dq), static_cast<TO *>(g.dk),
        static_cast<TO *>(g.dw), g.dbeta, sm_count(), saved, err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool prep_backward_ut_supported(const PrepDims &Dm, const PrepInputs &in)
{
    // the save area's stacked maps index up to 4 nh nblk 128 rows (int32)
    return prep_forward_ut_supported(Dm, in) && (long long)Dm.nh * Dm.nblk * 4 * BT < (1LL << 31);
}

cudaError_t prep_backward_ut(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g,
                             const UtSave &sv, const int *saved, int *err, cudaStream_t st)
{
    if (!prep_backward_ut_supported(Dm, in)) return cudaErrorInvalidValue;
    // What, U, X, M and Kta, Qtb, Pa, Pb lie back to back (carve_ut_save): one map each
    const uint64_t nb = (uint64_t)Dm.nh * Dm.nblk, hsz = nb * 2 * HB * HB, bsz = nb * HB * HB;
    if (sv.U != sv.What + hsz || sv.X != sv.U + hsz || sv.M != sv.X + hsz || sv.Qtb != sv.Kta + bsz ||
        sv.Pa != sv.Qtb + bsz || sv.Pb != sv.Pa + bsz)
        return cudaErrorInvalidValue;
    CUtensorMap m[5];
    if (!make_map_3d(&m[0], in.w, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[1], in.q, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[2], in.k, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_2d(&m[3], sv.What, F16, HB, 4 * nb * 2 * HB, HB) ||
        !make_map_2d(&m[4], sv.Kta, F16, HB, 4 * nb * HB, HB))
        return cudaErrorInvalidValue;
    if (Dm.odt == F32) return launch<float>(m, Dm, in, g, saved, err, st);
    return launch<bf16>(m, Dm, in, g, saved, err, st);
}

}  // namespace path
